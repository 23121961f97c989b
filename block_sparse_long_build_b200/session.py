"""Decode sessions: buffers and call sequence of the block-sparse decode path.

A session owns the device buffers one workload needs (summaries, selection
outputs, workspace) and issues the library calls of one decode step in
order:

    append (new K/V row; summary of a page that completes)   -- bsa_append_kv
    select (score + top-k/budget + ranges), every `refresh` steps -- bsa_select
    decode (split-K attention over the ranges + LSE merge)   -- bsa_decode

Steps that do not refresh the selection run append and decode as one call
(bsa_decode_step: one launch on the tensor-core path) unless `fused` is
False.

Everything here is allocation and sequencing; the arithmetic runs in
libbsa's kernels.
"""
from __future__ import annotations

import math

import torch

from . import native as N
from .workloads import Config, Workload


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class DecodeSession:
    """page_rows > 0 keeps the cache as a page pool (Workload.paged) instead
    of the workload's contiguous [B, Hkv, L_max, D] tensors."""

    def __init__(self, wl: Workload, stream: torch.cuda.Stream | None = None, fused: bool = True,
                 page_rows: int = 0, spare_pages: int = 0):
        self.wl = wl
        self.fused = fused
        c = self.cfg = wl.cfg
        dev = wl.device
        self.stream = stream
        if page_rows:
            self.K, self.V, self.page_table = wl.paged(page_rows, spare_pages)
            self.desc = N.paged_kv_desc(self.K, c.Hq, self.page_table)
        else:
            self.K, self.V, self.page_table = wl.K, wl.V, None
            self.desc = N.kv_desc(wl.K, c.Hq)
        if c.block_size == 0:
            self.sel = N.sel_params(0, c.n_blocks, wl.block_offsets, wl.kv_pos, topk=-1,
                                    budget_tokens=c.budget_tokens, local_start=wl.local_start,
                                    pos_limit=c.L - c.chunk)
        else:
            self.sel = N.sel_params(c.block_size, topk=c.topk, budget_tokens=c.budget_tokens,
                                    sink=c.sink, window=c.window,
                                    keep_current_block=c.keep_current)
        self.kind = c.kind
        nb = N.bsa_summary_blocks(self.desc, self.sel)
        assert nb > 0
        self.nb = nb
        sbytes = N.bsa_summary_bytes(self.desc, self.sel, self.kind)
        self.summaries = torch.zeros(sbytes, dtype=torch.uint8, device=dev)
        self.max_sel = N.bsa_max_selected(self.desc, self.sel)
        self.max_ranges = N.bsa_max_ranges(self.desc, self.sel)
        nseg = c.B * c.Hkv
        self.sel_blocks = torch.zeros(nseg, self.max_sel, dtype=torch.int32, device=dev)
        self.sel_count = torch.zeros(nseg, dtype=torch.int32, device=dev)
        self.ranges = torch.zeros(nseg, self.max_ranges, 2, dtype=torch.int32, device=dev)
        self.n_ranges = torch.zeros(nseg, dtype=torch.int32, device=dev)
        self.tokens_hint = self.token_bound()
        self.decode_kernels = N.bsa_decode_kernels(self.desc, self.sel, self.tokens_hint)
        ws = max(N.bsa_workspace_size(self.desc, self.sel, op, 0, self.tokens_hint)
                 for op in (N.BSA_OP_SELECT, N.BSA_OP_DECODE, N.BSA_OP_APPEND))
        self.ws = torch.zeros(ws, dtype=torch.uint8, device=dev)
        # outputs in one buffer (out, then lse) so a step's results leave the
        # device in one copy
        n_out = c.B * c.Hq * c.D * 4
        self.io_out = torch.zeros(_align(n_out) + c.B * c.Hq * 4, dtype=torch.uint8, device=dev)
        self.out = self.io_out[:n_out].view(torch.float32).view(c.B, c.Hq, c.D)
        self.lse = self.io_out[_align(n_out):].view(torch.float32).view(c.B, c.Hq)
        self.scale = 1.0 / math.sqrt(c.D)

    def token_bound(self) -> int:
        """Upper bound on the tokens one segment's ranges cover."""
        c = self.cfg
        if c.block_size == 0:
            return c.budget_tokens + c.chunk + c.steps + 1
        S = c.block_size
        k = self.max_sel
        return c.sink + c.window + k * S + S + c.refresh + 1

    # ----------------------------------------------------------------- steps
    def build_summaries(self, n_tokens: int | None = None):
        """Summaries of every block complete in the first n_tokens rows."""
        c = self.cfg
        if c.block_size == 0:
            nb = self.nb
        else:
            nb = (n_tokens if n_tokens is not None else c.L) // c.block_size
        N.bsa_build_summaries(self.desc, self.K, self.sel, self.kind, 0, nb, self.summaries,
                              self.stream)

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor):
        N.bsa_append_kv(self.desc, self.K, self.V, k_new, v_new, self.wl.cur_len, self.sel,
                        self.kind, self.summaries if self.cfg.block_size > 0 else None,
                        self.stream)

    def select(self, q: torch.Tensor):
        N.bsa_select(self.desc, q, self.summaries, self.kind, self.sel, self.wl.cur_len,
                     self.max_sel, self.sel_blocks, self.sel_count, self.max_ranges, self.ranges,
                     self.n_ranges, self.ws, self.stream)

    def decode(self, q: torch.Tensor, out: torch.Tensor | None = None,
               lse: torch.Tensor | None = None):
        N.bsa_decode(self.desc, q, self.K, self.V, self.ranges, self.n_ranges,
                     self.max_ranges, self.wl.cur_len, self.tokens_hint, self.scale,
                     self.out if out is None else out, self.lse if lse is None else lse,
                     self.ws, self.stream)

    def decode_step(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                    out: torch.Tensor | None = None, lse: torch.Tensor | None = None):
        """Append the new row and attend (no selection refresh)."""
        N.bsa_decode_step(self.desc, q, self.K, self.V, k_new, v_new, self.wl.cur_len,
                          self.sel, self.kind,
                          self.summaries if self.cfg.block_size > 0 else None, self.ranges,
                          self.n_ranges, self.max_ranges, self.tokens_hint, self.scale,
                          self.out if out is None else out, self.lse if lse is None else lse,
                          self.ws, self.stream)

    def step(self, t: int, q: torch.Tensor, k_new: torch.Tensor | None, v_new: torch.Tensor | None):
        """Decode step t: append (when new K/V are given), select on refresh
        steps, attend."""
        refresh = t % self.cfg.refresh == 0
        if k_new is not None and self.fused and not refresh:
            self.decode_step(q, k_new, v_new)
            return
        if k_new is not None:
            self.append(k_new, v_new)
        if refresh:
            self.select(q)
        self.decode(q)

    # ---------------------------------------------------------------- prefill
    def prefill_chunk(self, Q: torch.Tensor, q_pos0: int, out: torch.Tensor, lse: torch.Tensor,
                      ws: torch.Tensor | None = None) -> torch.Tensor:
        """Block-grouped prefill of the query rows Q [Tq, Hq, D] (bf16) at
        positions q_pos0.. of a semantic-block workload: dense causal while
        the prefix is shorter than the configured dense limit, otherwise the
        chunk densely and causally plus the blocks each query selects under a
        budget of 1/16 of the prefix.  Returns the workspace used."""
        c, wl = self.cfg, self.wl
        Tq = Q.shape[0]
        sparse = q_pos0 >= c.dense_below
        sel = N.sel_params(0, c.n_blocks, wl.block_offsets, wl.kv_pos, topk=-1,
                           budget_tokens=q_pos0 // 16 if sparse else 0,
                           local_start=wl.local_start, pos_limit=q_pos0 if sparse else 0)
        # the position-ordered window the local part reads: the chunk's own
        # rows past the dense limit, the whole prefix below it
        base = q_pos0 if sparse else 0
        Kw = wl.Kpos[:, :, base:q_pos0 + Tq]
        Vw = wl.Vpos[:, :, base:q_pos0 + Tq]
        pos_desc = N.kv_desc(Kw, c.Hq)
        need = N.bsa_workspace_size(self.desc, sel, N.BSA_OP_PREFILL, Tq, 0)
        if ws is None or ws.numel() < need:
            ws = torch.zeros(need, dtype=torch.uint8, device=wl.device)
        N.bsa_prefill_grouped(self.desc, wl.K, wl.V, sel, self.summaries, pos_desc, Kw, Vw, base,
                              Q, q_pos0, Tq, self.scale, out, lse, ws, self.stream)
        return ws

    # ------------------------------------------------------------ CUDA graphs
    def io_in_layout(self) -> tuple[int, int, int, int]:
        """Byte offsets of q, k_new, v_new in the packed step-input buffer, and
        its size (q fp32 [B, Hq, D], k_new / v_new in the cache dtype
        [B, Hkv, D], each 256-byte aligned)."""
        c = self.cfg
        esz = torch.empty(0, dtype=c.kv_dtype).element_size()
        nq, nk = c.B * c.Hq * c.D * 4, c.B * c.Hkv * c.D * esz
        ok = _align(nq)
        ov = ok + _align(nk)
        return 0, ok, ov, ov + _align(nk)

    def pack_inputs(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    pin: bool = True) -> torch.Tensor:
        """One step's inputs packed on the host in the layout of io_in (a
        single host-to-device copy feeds a step)."""
        oq, ok, ov, n = self.io_in_layout()
        buf = torch.zeros(n, dtype=torch.uint8)
        if pin:
            buf = buf.pin_memory()
        for o, x in ((oq, q), (ok, k), (ov, v)):
            x = x.detach().cpu().contiguous()
            nbytes = x.numel() * x.element_size()
            buf[o:o + nbytes].view(x.dtype).copy_(x.view(-1))
        return buf

    def capture(self):
        """Captures one decode step into two CUDA graphs (with and without
        the selection refresh) reading persistent input buffers q_in, k_in,
        v_in.  Launch-bound steps then cost one graph launch each.  Run one
        eager step first so that one-time host setup is not captured."""
        c, dev = self.cfg, self.wl.device
        oq, ok, ov, n = self.io_in_layout()
        esz = torch.empty(0, dtype=c.kv_dtype).element_size()
        nq, nk = c.B * c.Hq * c.D * 4, c.B * c.Hkv * c.D * esz
        self.io_in = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.q_in = self.io_in[oq:oq + nq].view(torch.float32).view(c.B, c.Hq, c.D)
        self.k_in = self.io_in[ok:ok + nk].view(c.kv_dtype).view(c.B, c.Hkv, c.D)
        self.v_in = self.io_in[ov:ov + nk].view(c.kv_dtype).view(c.B, c.Hkv, c.D)
        self.g_refresh, self.g_plain = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_refresh):
            self.append(self.k_in, self.v_in)
            self.select(self.q_in)
            self.decode(self.q_in)
        with torch.cuda.graph(self.g_plain):
            self._plain_step()
        # the same two steps with their host traffic inside the graph: the
        # packed inputs in from the pinned staging buffer host_in, the packed
        # outputs (out, lse) back to the pinned host_out
        self.host_in = torch.zeros(n, dtype=torch.uint8).pin_memory()
        self.host_out = torch.zeros(self.io_out.numel(), dtype=torch.uint8).pin_memory()
        self.g_refresh_io, self.g_plain_io = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_refresh_io):
            self.io_in.copy_(self.host_in, non_blocking=True)
            self.append(self.k_in, self.v_in)
            self.select(self.q_in)
            self.decode(self.q_in)
            self.host_out.copy_(self.io_out, non_blocking=True)
        with torch.cuda.graph(self.g_plain_io):
            self.io_in.copy_(self.host_in, non_blocking=True)
            self._plain_step()
            self.host_out.copy_(self.io_out, non_blocking=True)

    def _plain_step(self, q=None, k=None, v=None, out=None, lse=None):
        q = self.q_in if q is None else q
        k = self.k_in if k is None else k
        v = self.v_in if v is None else v
        if self.fused:
            self.decode_step(q, k, v, out, lse)
        else:
            self.append(k, v)
            self.decode(q, out, lse)

    def _io_views(self, io_in: torch.Tensor, io_out: torch.Tensor):
        c = self.cfg
        oq, ok, ov, _ = self.io_in_layout()
        esz = torch.empty(0, dtype=c.kv_dtype).element_size()
        nq, nk = c.B * c.Hq * c.D * 4, c.B * c.Hkv * c.D * esz
        q = io_in[oq:oq + nq].view(torch.float32).view(c.B, c.Hq, c.D)
        k = io_in[ok:ok + nk].view(c.kv_dtype).view(c.B, c.Hkv, c.D)
        v = io_in[ov:ov + nk].view(c.kv_dtype).view(c.B, c.Hkv, c.D)
        n_out = c.B * c.Hq * c.D * 4
        out = io_out[:n_out].view(torch.float32).view(c.B, c.Hq, c.D)
        lse = io_out[_align(n_out):].view(torch.float32).view(c.B, c.Hq)
        return q, k, v, out, lse

    def capture_pipelined(self):
        """Graphs for a pipelined step loop: two device input buffers and two
        output buffers (step t uses pair t % 2), so that a copy stream can
        bring step t+1's inputs in and take step t-1's outputs out while step
        t computes.  Four graphs: (refresh or not) x (buffer pair)."""
        dev = self.wl.device
        _, _, _, n = self.io_in_layout()
        self.pipe_in = [torch.zeros(n, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.pipe_out = [torch.zeros(self.io_out.numel(), dtype=torch.uint8, device=dev)
                         for _ in range(2)]
        self.g_pipe = {}
        for p in range(2):
            q, k, v, out, lse = self._io_views(self.pipe_in[p], self.pipe_out[p])
            for refresh in (True, False):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    if refresh:
                        self.append(k, v)
                        self.select(q)
                        self.decode(q, out, lse)
                    else:
                        self._plain_step(q, k, v, out, lse)
                self.g_pipe[(refresh, p)] = g

    def replay_pipelined(self, t: int):
        """Decode step t from buffer pair t % 2 (inputs already in pipe_in)."""
        self.g_pipe[(t % self.cfg.refresh == 0, t % 2)].replay()

    def replay(self, t: int):
        """Decode step t from the captured graphs (inputs already in q_in,
        k_in, v_in)."""
        (self.g_refresh if t % self.cfg.refresh == 0 else self.g_plain).replay()

    def replay_io(self, t: int):
        """Decode step t with its host traffic: the packed inputs staged in
        host_in (pinned) go in, the packed outputs come back to host_out, all in
        one graph launch."""
        (self.g_refresh_io if t % self.cfg.refresh == 0 else self.g_plain_io).replay()

    def launches_per_step(self, t: int) -> int:
        """Library kernels one step launches: append, the two selection kernels
        (scoring, picking) on refresh steps, and the decode (one kernel, or two
        when the split merge is a kernel of its own); a fused step folds the
        append into the decode."""
        if t % self.cfg.refresh == 0:
            return 3 + self.decode_kernels
        return self.decode_kernels + (0 if self.fused and self.fuses() else 1)

    def fuses(self) -> bool:
        """Whether bsa_decode_step runs as one launch for this workload."""
        c = self.cfg
        tc = (c.kv_dtype == torch.bfloat16 and c.D in (64, 128)) or \
            (c.kv_dtype == torch.float8_e4m3fn and c.D == 128)
        return tc and c.G <= 8 and not (c.block_size > 0 and self.kind == N.BSA_SUM_CENTROID_NORM)
