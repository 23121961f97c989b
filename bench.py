"""Benchmark: block-sparse long-context decode on B200.

Headline workload: large-batch decode in an 8B-model shape -- batch 64, 32
query / 8 KV heads, head_dim 128, bf16 cache of 32,768 clustered keys per
sequence, pages of 32 with min/max bounds, budget 8,192 tokens, sink 256,
window 512, selection every step (the largest configuration that fits one
GPU).  The default run adds, in the same JSON object under "also", one line
each for the Quest-style decode (batch 4, 65,536 tokens, refresh every 32
steps), the MoBA-style decode (131,072 tokens, blocks of 512, top-16), the
MSA-shaped decode, the semantic-block decode (524,288 tokens), the
block-grouped prefill of the 524,288-token semantic context and the semantic
index build.

One decode step = the whole hot path for the batch: append the new K/V row
(and the summary of a page it completes), select on refresh steps (score
every page, top-k under the budget, ranges), split-K attention over the
selected ranges with the log-sum-exp merge.  K steps are the configuration's
decode steps 0..K-1.

Timing: each step is one CUDA-graph replay bracketed by CUDA events on the
launching stream; between timed steps the L2 is flushed (a 512 MiB write and
a 512 MiB read), outside the events.  Throughput = tokens decoded / summed
step time; for N GPUs (torchrun) every rank decodes its own replica
(independent sequences, no collective on the data path) and the time is the
max over ranks.  e2e: the same steps with each step's packed inputs copied in
from pinned host memory and its packed outputs copied back, inside the
step's graph.  cpu_baseline: the CPU oracle on a bounded sample of the same
workload on the host cores; the same sample is compared with the GPU's
outputs of step 0 (parity_sample: selections bit for bit, outputs within
2e-3, near-ties counted).

Flags: --gpus N --steps K --warmup W [--impl reference] [--config NAME]
[--only] [--prefill] [--index] [--case NAME]
"""
from __future__ import annotations

import argparse
import gc
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
CSRC = os.path.join(ROOT, "block_sparse_long_build_b200", "csrc")
HEADLINE = "largebatch"
ALSO_DECODE = ("quest", "moba", "msa", "semantic", "largebatch_fp8", "quest_fp8")
DTYPE_NAMES = {torch.bfloat16: "bf16", torch.float32: "f32", torch.float8_e4m3fn: "e4m3"}
ATOL = 2e-3
L2_BYTES = 126 << 20      # B200 L2


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, burst copy)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def _bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (bf16_tflops_sustained)"
    return 1400.0, "fallback 1.4 PFLOP/s sustained"


def _sha(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def _profiled_traffic(profile: str, source: str):
    """DRAM bytes per launch (read + write) from a committed ncu summary, if
    it was taken on the current kernel source, else None."""
    path = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(path):
        return None
    sha = traffic = None
    for line in open(path).read().splitlines():
        if line.startswith("kernel_source_sha:"):
            sha = line.split(":", 1)[1].strip()
        if line.startswith("dram_bytes_per_launch:"):
            traffic = float(line.split(":", 1)[1].strip())
    return traffic if sha == _sha(os.path.join(CSRC, source)) else None


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


def _release(device):
    gc.collect()
    if device.type == "cuda":
        torch.cuda.synchronize(device)
        torch.cuda.empty_cache()


def _step_bytes(sess, t: int) -> tuple[int, int]:
    """Algorithmic bytes of step t (call after the step ran): K and V rows of
    the selected tokens, queries and outputs, and on refresh steps the page
    summaries the selection reads.  Returns (total, decode-kernel bytes)."""
    c = sess.cfg
    ranges = sess.ranges.cpu().numpy()
    nr = sess.n_ranges.cpu().numpy()
    cur = sess.wl.cur_len.cpu().numpy()
    esz = torch.empty(0, dtype=c.kv_dtype).element_size()
    sesz = 4 if c.kv_dtype == torch.float32 else 2   # min/max summaries: bf16 for bf16 and FP8
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
        row_bytes = 2 * c.D * sesz if c.kind == 2 else c.D * 4
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


def _workload_text(cfg, W) -> str:
    return f"{cfg.name}: " + " ".join((W.CONFIGS[cfg.name].__doc__ or "").split())


# ---------------------------------------------------------------- decode

def decode_line(name: str, K_steps: int, W_steps: int, rank: int, world: int, device,
                cpu_budget: float):
    """One decode configuration: the timed graph-replayed steps, the decode
    kernel alone (roofline), the end-to-end steps and the CPU baseline."""
    from block_sparse_long_build_b200 import native as N
    from block_sparse_long_build_b200 import workloads as W
    from block_sparse_long_build_b200.session import DecodeSession

    cfg = W.CONFIGS[name](0)
    cfg = cfg.scaled(steps=max(K_steps, W_steps, cfg.steps))
    wl = W.Workload(cfg, device)
    sess = DecodeSession(wl)
    sess.build_summaries()
    L0 = int(wl.cur_len[0].item())   # rows in each cache when decoding starts
    inputs = [(wl.decode_query(t), *wl.decode_new_kv(t)) for t in range(max(K_steps, W_steps))]
    torch.cuda.synchronize()

    # census: run the K steps once untimed to count each step's bytes; keep
    # step 0's results for the parity sample
    step_bytes, dec_bytes = [], []
    step0 = None
    for t in range(K_steps):
        q, k, v = inputs[t]
        sess.step(t, q, k, v)
        tb, db = _step_bytes(sess, t)
        step_bytes.append(tb)
        dec_bytes.append(db)
        if t == 0:
            step0 = {"out": sess.out.cpu().numpy().copy(), "lse": sess.lse.cpu().numpy().copy(),
                     "sel": sess.sel_blocks.cpu().numpy().copy(),
                     "cnt": sess.sel_count.cpu().numpy().copy(), "n": L0 + 1}
    st, bits = N.bsa_workspace_status(sess.ws)
    assert st == N.BSA_OK, f"device status {bits:#x} after the census steps"
    out_census = sess.out.clone()

    def reset():
        wl.cur_len.fill_(L0)

    # graphs
    reset()
    sess.step(0, *inputs[0])      # one eager step: one-time host setup
    reset()
    sess.capture()
    if min(step_bytes) > 2 * L2_BYTES:
        sess.capture_pipelined()
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
    # the graph-replayed steps reproduce the eager census bit for bit
    assert torch.equal(sess.out, out_census), "replayed steps differ from the eager census"
    st, bits = N.bsa_workspace_status(sess.ws)
    assert st == N.BSA_OK, f"device status {bits:#x} after the timed steps"
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
    # the last step's results reached the host, equal to the device's
    assert torch.equal(sess.host_out, sess.io_out.cpu()), "host outputs differ from the device's"
    assert torch.equal(sess.out, out_census), "end-to-end steps differ from the eager census"
    h2d = pin_in[0].numel()
    d2h = sess.host_out.numel()
    e2e_path = ("per step, one graph launch: the step's packed inputs from a pinned host buffer "
                "-> device, the step's kernels, the packed outputs -> pinned host; L2 flushed "
                "between steps outside the events")
    e2e_serial = None
    if min(step_bytes) > 2 * L2_BYTES:
        # every step reads more than the L2 holds: the steps run back to back in
        # one timed region, each step's inputs copied in (copy stream) while the
        # previous step computes and its outputs copied out while the next
        # computes -- every copy of every step inside the region
        e2e_serial = world * cfg.B * K_steps / (e2e_ms / 1e3)
        e2e_ms = _pipelined_e2e_ms(sess, pin_in, K_steps, reset, out_census)
        e2e_ms = max_over_ranks(e2e_ms, device, world)
        e2e_path = ("all steps back to back in one timed region: step t+1's packed inputs copied "
                    "in from pinned host memory on a copy stream while step t computes, step t's "
                    "packed outputs copied out to pinned host memory on a second stream while "
                    "step t+1 computes (two device buffer pairs); the step reads more than twice "
                    "the L2, so no flush is needed")

    launches = sum(sess.launches_per_step(t) for t in range(K_steps))
    decode_kernel = ("decode_tc_kernel (split-K sparse decode, split merge inside a thread-block "
                     "cluster)" if sess.decode_kernels == 1 else
                     "decode_tc_kernel + lse_merge_kernel (split-K sparse decode, then the merge)")
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
        "dtype": DTYPE_NAMES[cfg.kv_dtype],
        "data": "synthetic",
        "effective_kv_gbs": eff_gbs,
        "effective_kv_frac_of_8tbs": eff_gbs / 8000.0,
        "config": {
            "workload": _workload_text(cfg, W),
            "global_batch": cfg.B * world,
            "seq_len": cfg.L,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed between timed steps (512 MiB write + 512 MiB read, outside the events)",
            "timing": "CUDA events per graph-replayed step on the launching stream",
        },
        "roofline": {
            "kernel": f"bsa_decode: {decode_kernel}",
            "bound": "hbm",
            "achieved": achieved,
            "peak": peak,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": achieved / peak,
            "frac_of_8tbs": achieved / 8000.0,
            "traffic": _profiled_traffic(f"decode_tc_{cfg.name}.md", "decode.cu"),
            "algorithmic_bytes_per_launch": kbytes,
            "launch_ms": k_ms,
        },
        "clocks": clocks,
        "e2e": {"value": world * cfg.B * K_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "path": e2e_path,
                "serial_value": e2e_serial},
        "gpu_launches": launches,
    }
    if rank == 0 and world == 1 and cpu_budget > 0:
        res["cpu_baseline"], res["parity_sample"] = cpu_baseline_decode(
            cfg, wl, inputs[0], step0, cpu_budget)
    del sess, wl, inputs
    return res


def _pipelined_e2e_ms(sess, pin_in, K_steps, reset, out_census) -> float:
    """K steps in one timed region with the host copies overlapped: inputs of
    step t+1 in (stream cin) while step t computes, outputs of step t out
    (stream cout) while step t+1 computes.  Buffer pair t % 2 carries step t;
    events order every reuse.  Returns the region's milliseconds."""
    main = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    hout = [torch.empty(sess.pipe_out[0].numel(), dtype=torch.uint8).pin_memory() for _ in range(2)]
    ev = lambda: torch.cuda.Event()
    in_ev, comp_ev, out_ev = ([ev() for _ in range(K_steps)] for _ in range(3))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def h2d(t):
        with torch.cuda.stream(cin):
            if t >= 2:
                cin.wait_event(comp_ev[t - 2])   # step t-2 has read this buffer
            sess.pipe_in[t % 2].copy_(pin_in[t], non_blocking=True)
            in_ev[t].record(cin)

    reset()
    torch.cuda.synchronize()
    start.record(main)
    cin.wait_event(start)
    h2d(0)
    for t in range(K_steps):
        if t + 1 < K_steps:
            h2d(t + 1)
        main.wait_event(in_ev[t])
        if t >= 2:
            main.wait_event(out_ev[t - 2])       # step t-2's outputs have left this buffer
        sess.replay_pipelined(t)
        comp_ev[t].record(main)
        with torch.cuda.stream(cout):
            cout.wait_event(comp_ev[t])
            hout[t % 2].copy_(sess.pipe_out[t % 2], non_blocking=True)
            out_ev[t].record(cout)
    main.wait_event(out_ev[K_steps - 1])
    end.record(main)
    torch.cuda.synchronize()
    last = hout[(K_steps - 1) % 2]
    n_out = out_census.numel() * 4
    got = last[:n_out].view(torch.float32).view(out_census.shape)
    assert torch.equal(got, out_census.cpu()), "pipelined steps differ from the eager census"
    return start.elapsed_time(end)


def _host(t):
    """bf16 as uint16 bit patterns, FP8 as uint8 codes, fp32 as float32."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def _oracle_kv(a):
    """FP8 codes decoded by the oracle's own E4M3 table (it reads fp32 or
    bf16 bits); other arrays as they are."""
    import oracle
    return oracle.fp8_e4m3_to_f32(a) if a.dtype == np.uint8 else a


def _host_cores() -> int:
    return os.cpu_count() or 1


def _sample_segments(cfg, n_max=64):
    segs = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    if len(segs) <= n_max:
        return segs
    rng = np.random.default_rng(7)
    return [segs[i] for i in sorted(rng.choice(len(segs), n_max, replace=False))]


def cpu_baseline_decode(cfg, wl, inputs0, step0, budget_s):
    """The oracle's decode step (summaries, scores, selection and fp64
    attention of one (sequence, KV head) segment per call, single thread) on a
    bounded sample of step 0's segments, scaled to one step of the batch; the
    same calls are compared with the GPU's step-0 results."""
    import oracle
    oracle.build()
    q0 = _host(inputs0[0])
    n = step0["n"]
    segs = _sample_segments(cfg)
    semantic = cfg.block_size == 0
    if semantic:
        Kpos, Vpos = _host(wl.Kpos), _host(wl.Vpos)
        Kpos[0, :, cfg.L] = _host(inputs0[1])[0]
        Vpos[0, :, cfg.L] = _host(inputs0[2])[0]
        labels = wl.labels.cpu().numpy()
        local0 = cfg.L - cfg.chunk
    done, t_acc, ties, sel_equal, worst = 0, 0.0, 0, True, 0.0
    for b, g in segs:
        qg = q0[b, g * cfg.G:(g + 1) * cfg.G]
        s = b * cfg.Hkv + g
        if semantic:
            lab = labels[b, g]
            t0 = time.perf_counter()
            sel, pos, tie, _ = oracle.semantic_select_positions(
                qg, Kpos[b, g, :cfg.L], lab, cfg.n_blocks, local0, cfg.budget_tokens)
            rows = np.concatenate([pos, np.arange(local0, cfg.L + 1)])
            out, lse = oracle.attend(qg, Kpos[b, g], Vpos[b, g], rows, 1 / math.sqrt(cfg.D))
            t_acc += time.perf_counter() - t0
        else:
            K, V = _oracle_kv(_host(wl.K[b, g])), _oracle_kv(_host(wl.V[b, g]))
            t0 = time.perf_counter()
            ref = oracle.decode_fixed_segment(qg, K, V, n, n, cfg.kind, cfg.block_size, cfg.topk,
                                              cfg.budget_tokens, cfg.sink, cfg.window,
                                              cfg.keep_current, 1 / math.sqrt(cfg.D))
            t_acc += time.perf_counter() - t0
            sel, tie, out, lse = ref["sel"], ref["ties"], ref["out"], ref["lse"]
        done += 1
        ties += len(tie)
        sel_equal &= step0["sel"][s, :step0["cnt"][s]].tolist() == list(sel)
        worst = max(worst, float(np.abs(step0["out"][b, g * cfg.G:(g + 1) * cfg.G] - out).max()),
                    float(np.abs(step0["lse"][b, g * cfg.G:(g + 1) * cfg.G] - lse).max()))
        if t_acc >= budget_s:
            break
    per_step = t_acc / done * cfg.B * cfg.Hkv
    base = {"value": cfg.B / per_step, "unit": "tokens/s", "cores": 1, "host_cores": _host_cores(),
            "kind": "oracle",
            "sample": f"{done} of the {cfg.B * cfg.Hkv} (sequence, KV head) segments of step 0, "
                      f"one oracle decode step each on one thread (summaries, scores, selection, "
                      f"fp64 attention), scaled to one {cfg.B}-sequence step"}
    parity = {"segments": done, "step": 0, "selection_bit_exact": bool(sel_equal),
              "max_abs_err": worst, "tolerance": ATOL, "pass": bool(sel_equal and worst <= ATOL),
              "near_tie_pairs": ties}
    return base, parity


# ---------------------------------------------------------------- prefill

def prefill_line(device, cpu_budget: float, context: int = 0):
    """Block-grouped prefill of the semantic-block configuration: every
    4096-query chunk of the 524,288-token context (dense while the prefix is
    under 16k), one bsa_prefill_grouped call per chunk, each timed with CUDA
    events; L2 is flushed before each chunk.  e2e: all chunks in one timed
    region, each chunk's queries copied in from pinned host memory and its
    outputs copied back, the copies overlapped with the neighbouring chunks'
    calls (serial_value: one chunk at a time)."""
    from block_sparse_long_build_b200 import native as N
    from block_sparse_long_build_b200 import workloads as W
    from block_sparse_long_build_b200.session import DecodeSession

    cfg = W.semantic(0)
    if context:
        cfg = cfg.scaled(L=context, budget_tokens=context // 16)
    wl = W.Workload(cfg, device)
    sess = DecodeSession(wl)
    sess.build_summaries()
    Tq = cfg.chunk
    out_all = torch.empty(cfg.L, cfg.Hq, cfg.D, dtype=torch.float32, device=device)
    lse_all = torch.empty(cfg.L, cfg.Hq, dtype=torch.float32, device=device)
    flush = _flusher(device)
    chunks = list(range(0, cfg.L, Tq))
    times, pairs = [], 0
    # warm-up on the first sparse chunk (one-time host setup, caches)
    warm = next((p for p in chunks if p >= cfg.dense_below), 0)
    ws = sess.prefill_chunk(wl.prefill_queries(warm, Tq), warm, out_all[:Tq], lse_all[:Tq], None)
    torch.cuda.synchronize()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    for p in chunks:
        n = min(Tq, cfg.L - p)
        Q = wl.prefill_queries(p, n)
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ws = sess.prefill_chunk(Q, p, out_all[p:p + n], lse_all[p:p + n], ws)
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
            bits = ((words.unsqueeze(-1) >> torch.arange(32, device=device)) & 1).reshape(
                n, cfg.Hkv, 256)
            vis_off = cb + n * cfg.Hkv * 8 * 4
            vis_off = (vis_off + 255) // 256 * 256
            vis = ws[vis_off:vis_off + cfg.Hkv * cfg.n_blocks * 4].view(torch.int32).view(
                cfg.Hkv, cfg.n_blocks)
            grouped = int((bits[:, :, :cfg.n_blocks].long() * vis.long()[None]).sum().item()) * cfg.G
        pairs += local + grouped
    clocks = sampler.stop()
    st, bits = N.bsa_workspace_status(ws)
    assert st == N.BSA_OK, f"prefill device status {bits:#x}"
    total_ms = float(sum(times))
    flops = 4.0 * pairs * cfg.D
    tflops = flops / (total_ms / 1e3) / 1e12
    peak = _bf16_peak()

    # e2e, one chunk at a time (serial_value): each chunk's queries from a
    # pinned host buffer, the call, its outputs back; L2 flushed before each
    q_host = torch.empty(Tq, cfg.Hq, cfg.D, dtype=torch.bfloat16).pin_memory()
    o_host = torch.empty(Tq, cfg.Hq, cfg.D, dtype=torch.float32).pin_memory()
    l_host = torch.empty(Tq, cfg.Hq, dtype=torch.float32).pin_memory()
    q_dev = torch.empty(Tq, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=device)
    serial_ms = 0.0
    for p in chunks:
        n = min(Tq, cfg.L - p)
        q_host[:n].copy_(wl.prefill_queries(p, n).cpu())
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        q_dev[:n].copy_(q_host[:n], non_blocking=True)
        ws = sess.prefill_chunk(q_dev[:n], p, out_all[p:p + n], lse_all[p:p + n], ws)
        o_host[:n].copy_(out_all[p:p + n], non_blocking=True)
        l_host[:n].copy_(lse_all[p:p + n], non_blocking=True)
        e1.record()
        e1.synchronize()
        serial_ms += e0.elapsed_time(e1)
    assert torch.equal(o_host[:Tq].to(device), out_all[chunks[-1]:chunks[-1] + Tq])
    del q_host, o_host, l_host, q_dev

    # e2e: every chunk's queries from pinned host memory and its outputs and
    # log-sum-exp back to pinned host memory, all inside one timed region.
    # Chunks are independent (a prompt's queries are all known), so chunk
    # i+1's queries go up on one copy stream and chunk i's outputs come down
    # on another while chunk i+1 computes; each chunk reads far more than the
    # L2 holds, so the chunks run back to back without a flush.
    q_all = torch.empty(cfg.L, cfg.Hq, cfg.D, dtype=torch.bfloat16, pin_memory=True)
    for p in chunks:
        n = min(Tq, cfg.L - p)
        q_all[p:p + n].copy_(wl.prefill_queries(p, n))
    comp = torch.cuda.current_stream(device)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    q_dev2 = [torch.empty(Tq, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=device) for _ in range(2)]
    o_ring = [torch.empty(Tq, cfg.Hq, cfg.D, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    l_ring = [torch.empty(Tq, cfg.Hq, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    ev_up = [torch.cuda.Event() for _ in chunks]
    ev_done = [torch.cuda.Event() for _ in chunks]
    ev_down = [torch.cuda.Event() for _ in chunks]
    out_all.zero_()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    n0 = min(Tq, cfg.L)
    with torch.cuda.stream(up):
        q_dev2[0][:n0].copy_(q_all[:n0], non_blocking=True)
        ev_up[0].record(up)
    for i, p in enumerate(chunks):
        n = min(Tq, cfg.L - p)
        if i + 1 < len(chunks):
            p1 = chunks[i + 1]
            n1 = min(Tq, cfg.L - p1)
            if i >= 1:
                up.wait_event(ev_done[i - 1])   # chunk i-1 has read buffer (i+1) & 1
            with torch.cuda.stream(up):
                q_dev2[(i + 1) & 1][:n1].copy_(q_all[p1:p1 + n1], non_blocking=True)
                ev_up[i + 1].record(up)
        comp.wait_event(ev_up[i])
        ws = sess.prefill_chunk(q_dev2[i & 1][:n], p, out_all[p:p + n], lse_all[p:p + n], ws)
        ev_done[i].record(comp)
        down.wait_event(ev_done[i])
        with torch.cuda.stream(down):   # ring slot i & 1: chunk i-2's copy came first on this stream
            o_ring[i & 1][:n].copy_(out_all[p:p + n], non_blocking=True)
            l_ring[i & 1][:n].copy_(lse_all[p:p + n], non_blocking=True)
            ev_down[i].record(down)
    comp.wait_event(ev_down[-1])
    e1.record(comp)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    last = chunks[-1]
    nl = min(Tq, cfg.L - last)
    assert torch.equal(o_ring[(len(chunks) - 1) & 1][:nl].to(device), out_all[last:last + nl])
    assert torch.equal(l_ring[(len(chunks) - 1) & 1][:nl].to(device), lse_all[last:last + nl])
    del q_all, o_ring, l_ring, q_dev2
    res = {
        "metric": "block-grouped prefill tokens/s (semantic blocks); roofline on algorithmic "
                  "TFLOP/s = 4 x attended (query head, key) pairs x head_dim",
        "value": cfg.L / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": len(chunks), "warmup": 1, "ms_total": total_ms,
        "ms_per_step": total_ms / len(chunks), "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic", "algorithmic_tflop": flops / 1e12, "algorithmic_tflops": tflops,
        "config": {"workload": f"semantic blocks prefill: batch 1, {cfg.Hkv} KV / {cfg.Hq} query "
                               f"heads, head_dim {cfg.D}, context {cfg.L}, {cfg.n_blocks} blocks, "
                               f"chunks of {Tq}, dense below {cfg.dense_below}, budget prefix/16",
                   "l2": "flushed before each chunk"},
        "roofline": {"kernel": "prefill_attend_kernel + prefill_select_kernel + prefill_merge_kernel "
                               "(whole call; the tcgen05 contraction dominates)",
                     "bound": "tensor", "achieved": tflops, "peak": peak[0], "unit": "TFLOP/s",
                     "frac": tflops / peak[0], "peak_source": peak[1],
                     "traffic": None},
        "clocks": clocks,
        "e2e": {"value": cfg.L / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": Tq * cfg.Hq * cfg.D * 2,
                "d2h_bytes_per_step": Tq * cfg.Hq * (cfg.D + 1) * 4,
                "serial_value": cfg.L / (serial_ms / 1e3),
                "path": "every chunk in one timed region: its queries from pinned host memory -> "
                        "device on a copy stream (one chunk ahead), the prefill call, its outputs "
                        "and log-sum-exp -> pinned host on a second copy stream (overlapping the "
                        "next chunk); serial_value: one chunk at a time, L2 flushed before each"},
        "gpu_launches": 4 * len(chunks),
    }
    if cpu_budget > 0:
        res["cpu_baseline"], res["parity_sample"] = cpu_baseline_prefill(
            cfg, wl, out_all, lse_all, cpu_budget)
    del sess, wl, out_all, lse_all
    return res


def cpu_baseline_prefill(cfg, wl, out_all, lse_all, budget_s):
    """The oracle's prefill of single query rows (per KV head: block scores,
    greedy budget walk, fp64 attention over the selected and local rows; all
    heads of the row), rows drawn across the whole context, on one thread;
    tokens/s = rows per second.  The same rows are compared with the GPU's."""
    import oracle
    oracle.build()
    Kpos, Vpos = _host(wl.Kpos), _host(wl.Vpos)
    labels = wl.labels.cpu().numpy()
    Tq = cfg.chunk
    rng = np.random.default_rng(11)
    rows = rng.integers(0, cfg.L, 64)
    qs = {}
    done, t_acc, ties, sel_checked, worst = 0, 0.0, 0, 0, 0.0
    for r in rows.tolist():
        p = r // Tq * Tq
        if p not in qs:
            qs[p] = _host(wl.prefill_queries(p, min(Tq, cfg.L - p)))
        qrow = qs[p][r - p]
        sparse = p >= cfg.dense_below
        t0 = time.perf_counter()
        outs, lses = [], []
        for g in range(cfg.Hkv):
            qg = oracle.bf16_bits_to_f32(qrow[g * cfg.G:(g + 1) * cfg.G])
            if sparse:
                _, pos, tie, _ = oracle.semantic_select_positions(
                    qg, Kpos[0, g, :cfg.L], labels[0, g], cfg.n_blocks, p, p // 16)
                ties += len(tie)
                rws = np.concatenate([pos, np.arange(p, r + 1)])
            else:
                rws = np.arange(0, r + 1)
            o, l_ = oracle.attend(qg, Kpos[0, g], Vpos[0, g], rws, 1 / math.sqrt(cfg.D))
            outs.append(o)
            lses.append(l_)
        t_acc += time.perf_counter() - t0
        done += 1
        got_o = out_all[r].cpu().numpy()
        got_l = lse_all[r].cpu().numpy()
        worst = max(worst, float(np.abs(got_o - np.concatenate(outs)).max()),
                    float(np.abs(got_l - np.concatenate(lses)).max()))
        sel_checked += cfg.Hkv if sparse else 0
        if t_acc >= budget_s:
            break
    base = {"value": done / t_acc, "unit": "tokens/s", "cores": 1, "host_cores": _host_cores(),
            "kind": "oracle",
            "sample": f"{done} query rows drawn across the {cfg.L}-token context, every KV head "
                      f"(selection + fp64 attention), one thread"}
    parity = {"rows": done, "max_abs_err": worst, "tolerance": ATOL, "pass": worst <= ATOL,
              "near_tie_pairs": ties, "selections_sampled": sel_checked}
    return base, parity


# ---------------------------------------------------------------- index

def index_line(device, cpu_budget: float, keys: int = 0, warmup: int = 1, runs: int = 3):
    """The semantic index of the semantic-block configuration: spherical
    k-means over every KV head's 524,288 position-ordered keys (256 clusters,
    20 assignment rounds, one starting key per planted cluster) and the
    block-ordered store gathered from it, one bsa_build_semantic_index call
    plus one bsa_gather_rows call per run, timed with CUDA events after a
    warm-up run."""
    from block_sparse_long_build_b200 import native as N
    from block_sparse_long_build_b200 import workloads as W

    cfg = W.semantic(0)
    if keys:
        cfg = cfg.scaled(L=keys, budget_tokens=keys // 16)
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

    def run(keys_src):
        N.bsa_build_semantic_index(src, keys_src, L, k, iters, init, C, labels, offsets, order, ws)
        N.bsa_gather_rows(src, keys_src, wl.Vpos, dst, Kb, Vb, order, L, 0)

    for _ in range(max(1, warmup)):
        run(wl.Kpos)
    torch.cuda.synchronize()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    times = []
    for _ in range(max(1, runs)):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run(wl.Kpos)
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

    # e2e: the keys from pinned host memory, the index (labels, offsets,
    # order) back to pinned host memory
    k_host = wl.Kpos.cpu().pin_memory()
    k_dev = torch.empty_like(wl.Kpos)
    idx_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (labels, offsets, order)]
    flush()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    k_dev.copy_(k_host, non_blocking=True)
    run(k_dev)
    for h, d in zip(idx_host, (labels, offsets, order)):
        h.copy_(d, non_blocking=True)
    e1.record()
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    res = {
        "metric": "semantic index build (spherical k-means + block-ordered store), keys per second",
        "value": nseg * L / (ms / 1e3), "unit": "keys/s", "n_gpus": 1, "steps": len(times),
        "warmup": max(1, warmup), "ms_per_step": ms, "higher_is_better": True,
        "dtype": "f32", "data": "synthetic", "planted_clusters_recovered": recovered,
        "config": {"workload": f"semantic blocks index: {nseg} KV heads x {L} keys, head_dim {D}, "
                               f"bf16 keys, {k} clusters, {iters} assignment rounds",
                   "l2": "flushed before each run"},
        "roofline": {"kernel": "km_assign_tiled_kernel (whole call)", "bound": "alu",
                     "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                     "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flops x SM clock",
                     "traffic": None},
        "clocks": clocks,
        "e2e": {"value": nseg * L / (e2e_ms / 1e3), "unit": "keys/s",
                "h2d_bytes_per_step": k_host.numel() * k_host.element_size(),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in idx_host),
                "path": "keys from a pinned host buffer -> device, index build + store gather, "
                        "labels, offsets and order -> pinned host"},
        "gpu_launches": None,
    }
    if cpu_budget > 0:
        res["cpu_baseline"] = cpu_baseline_index(cfg, wl, cpu_budget)
    del wl, Kb, Vb, k_host, k_dev
    return res


def cpu_baseline_index(cfg, wl, budget_s):
    """The oracle's spherical k-means (20 rounds, 256 clusters) on the first
    keys of one KV head, growing the sample while it stays within the
    budget; keys/s over all KV heads."""
    import oracle
    oracle.build()
    K = _host(wl.Kpos[0, 0, :cfg.L])
    k, iters = cfg.n_blocks, 20
    n, rate = 1024, None
    while True:
        rng = np.random.default_rng(3)
        init = rng.choice(n, k, replace=False).astype(np.int32)
        t0 = time.perf_counter()
        oracle.spherical_kmeans(np.ascontiguousarray(K[:n]), k, iters, init)
        dt = time.perf_counter() - t0
        rate = n / dt
        if dt * 2.2 > budget_s or 2 * n > cfg.L:
            break
        n *= 2
    return {"value": rate, "unit": "keys/s", "cores": 1, "host_cores": _host_cores(),
            "kind": "oracle",
            "sample": f"spherical k-means of the first {n} keys of one KV head ({k} clusters, "
                      f"{iters} rounds), one thread; the rate scales with the keys"}


# ---------------------------------------------------------------- reference

def run_reference(args):
    """The oracle as it stands, on the host cores, same config and metric."""
    from block_sparse_long_build_b200 import workloads as W
    import oracle
    oracle.build()
    cfg = W.CONFIGS[args.config](0)
    wl = W.Workload(cfg, "cpu")
    n_total = args.warmup + args.steps
    per_step_budget = max(0.05, min(1.0, 150.0 / max(n_total, 1)))
    segs = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    times = []
    for t in range(n_total):
        q = _host(wl.decode_query(t))
        done, t_acc, i = 0, 0.0, t
        while True:
            b, g = segs[i % len(segs)]
            K, V = _oracle_kv(_host(wl.K[b, g])), _oracle_kv(_host(wl.V[b, g]))
            t0 = time.perf_counter()
            oracle.decode_fixed_segment(q[b, g * cfg.G:(g + 1) * cfg.G], K, V, cfg.L, cfg.L,
                                        cfg.kind, cfg.block_size, cfg.topk, cfg.budget_tokens,
                                        cfg.sink, cfg.window, cfg.keep_current, 1 / math.sqrt(cfg.D))
            t_acc += time.perf_counter() - t0
            done += 1
            i += 7
            if t_acc >= per_step_budget or done >= len(segs):
                break
        if t >= args.warmup:
            times.append(t_acc / done * len(segs))
    per_step = sum(times) / len(times)
    value = cfg.B / per_step
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name} (same as the CUDA arm)", "global_batch": cfg.B,
                   "seq_len": cfg.L, "parallelism": "host cores, one thread"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1,
                         "host_cores": _host_cores(), "kind": "oracle",
                         "sample": "each step: the oracle's per-segment decode step on a bounded "
                                   "sample of (sequence, KV head) segments, scaled to the batch"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- profiling cases

def run_case(args, device):
    """A small, fixed invocation of one library call for a profiler to capture
    (a few launches on a workload of a few GB at most); prints one line.
      decode      Quest workload (another with --case-config): two steps (the
                  second a fused append + decode where the workload fuses),
                  then bsa_decode five times, L2 flushed before each
      decode_lb   large-batch workload cut to --case-batch sequences (default
                  8: 1.1 GB of cache): one step, then bsa_decode five times, L2
                  flushed before each
      select      Quest workload (another with --case-config): bsa_select three
                  times, L2 flushed before each
      select_lb   large-batch workload cut to --case-batch sequences: bsa_select
                  three times
      prefill     semantic workload at a 65,536-token context (--case-context),
                  256 blocks (--case-blocks): the last chunk of 1,024 queries
                  (--case-chunk) three times"""
    from block_sparse_long_build_b200 import build as Bld
    from block_sparse_long_build_b200 import workloads as W
    from block_sparse_long_build_b200.session import DecodeSession
    Bld.build()
    flush = _flusher(device)
    ev = []
    if args.case in ("decode", "select", "decode_lb", "select_lb"):
        cfg = (W.CONFIGS[args.case_config](0) if args.case in ("decode", "select")
               else W.largebatch(0).scaled(B=args.case_batch))
        if args.case_fp8:
            cfg = cfg.scaled(kv_dtype=torch.float8_e4m3fn)
        wl = W.Workload(cfg, device)
        sess = DecodeSession(wl)
        sess.build_summaries()
        q = wl.decode_query(0)
        if args.case.startswith("decode"):
            for t in range(2):
                q = wl.decode_query(t)
                k, v = wl.decode_new_kv(t)
                sess.step(t, q, k, v)
        else:
            sess.step(0, q, *wl.decode_new_kv(0))
        for i in range(5 if args.case.startswith("decode") else 3):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sess.decode(q) if args.case.startswith("decode") else sess.select(q)
            e1.record()
            ev.append((e0, e1))
    elif args.case == "prefill":
        L, Tq = args.case_context, args.case_chunk
        cfg = W.semantic(0).scaled(L=L, budget_tokens=L // 16, chunk=Tq, n_blocks=args.case_blocks)
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


def _compact(line: dict) -> dict:
    """A secondary line without the keys it shares with the headline."""
    keep = ("metric", "value", "unit", "dtype", "steps", "warmup", "ms_per_step", "ms_total",
            "effective_kv_gbs", "effective_kv_frac_of_8tbs", "algorithmic_tflops",
            "planted_clusters_recovered", "config", "roofline", "e2e", "gpu_launches",
            "cpu_baseline", "parity_sample", "clocks")
    out = {k: line[k] for k in keep if k in line}
    if "config" in out:
        out["config"] = {"workload": out["config"]["workload"]}
    if "clocks" in out:
        c = out["clocks"]
        out["clocks"] = {"sm_mhz": c.get("sm_mhz"), "reasons": c.get("reasons")}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="decode steps to time (default: the configuration's own count, at most 64)")
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=None,
                    help="tiny | quest | moba | largebatch | semantic | msa: time this decode "
                         "configuration alone (default: large batch, plus the others under 'also')")
    ap.add_argument("--only", action="store_true",
                    help="the headline line alone, without the secondary lines")
    ap.add_argument("--prefill", action="store_true",
                    help="time the block-grouped prefill of the semantic configuration alone")
    ap.add_argument("--prefill-context", type=int, default=0,
                    help="context of the prefill run (default: the configuration's 524,288)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU-baseline budget of the headline line (secondary lines: a third)")
    ap.add_argument("--index", action="store_true",
                    help="time the semantic index build (k-means + block-ordered store) alone")
    ap.add_argument("--index-keys", type=int, default=0,
                    help="keys per KV head for --index (a smaller case for profiling)")
    ap.add_argument("--case", choices=["decode", "select", "decode_lb", "select_lb", "prefill"],
                    default=None, help="run one small profiling case instead of the bench (for ncu)")
    ap.add_argument("--case-config", default="quest",
                    help="decode / select cases: the decode configuration (quest, moba, msa, "
                         "semantic, ...)")
    ap.add_argument("--case-batch", type=int, default=8,
                    help="sequences of the large-batch profiling cases")
    ap.add_argument("--case-context", type=int, default=65536, help="prefill case: context length")
    ap.add_argument("--case-chunk", type=int, default=1024, help="prefill case: queries per chunk")
    ap.add_argument("--case-blocks", type=int, default=256, help="prefill case: semantic blocks")
    ap.add_argument("--case-fp8", action="store_true",
                    help="the decode and select profiling cases on an FP8 cache")
    args = ap.parse_args()
    if args.case:
        torch.cuda.set_device(0)
        run_case(args, torch.device("cuda", 0))
        return 0
    if args.warmup < 3:
        args.warmup = 3
    name = args.config or HEADLINE
    if args.steps is None:
        from block_sparse_long_build_b200 import workloads as W
        args.steps = min(64, W.CONFIGS[name](0).steps)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    cpu_s = 0.0 if args.no_cpu_baseline else args.cpu_seconds
    if args.impl == "reference":
        if rank == 0:
            args.config = name
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    from block_sparse_long_build_b200 import build as Bld
    if args.prefill or args.index:
        if rank == 0:
            Bld.build()
            res = (prefill_line(device, cpu_s, args.prefill_context) if args.prefill else
                   index_line(device, cpu_s, args.index_keys, args.warmup, args.steps))
            print(json.dumps(res), flush=True)
        return 0
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        if rank == 0:
            Bld.build()
        if world > 1:
            torch.distributed.barrier()
        res = decode_line(name, args.steps, args.warmup, rank, world, device, cpu_s)
        _release(device)
        if world == 1 and args.config is None and not args.only:
            also = []
            for other in ALSO_DECODE:
                from block_sparse_long_build_b200 import workloads as W
                steps = min(W.CONFIGS[other](0).steps, 128)
                also.append(_compact(decode_line(other, steps, args.warmup, 0, 1, device,
                                                 cpu_s / 3)))
                _release(device)
            also.append(_compact(prefill_line(device, cpu_s / 3)))
            _release(device)
            also.append(_compact(index_line(device, cpu_s / 3)))
            _release(device)
            res["also"] = also
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
