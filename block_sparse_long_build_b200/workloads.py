"""Seeded synthetic workloads for block-sparse long-context attention.

This module only draws inputs: KV caches, queries and the per-step new
tokens, with the shapes, distributions and structure of the workloads the
source pages measure (needle-in-a-haystack, clustered keys, long contexts).
It holds none of the method's arithmetic (no summaries, scores, selection or
attention) and is shared, as the only common code, by the CUDA path's tests,
the benchmark and the CPU oracle's tests.

Every random draw comes from a ``torch.Generator`` seeded from the config's
seed; step ``t``'s inputs come from seed + 1 + t.  The same call on the same
device returns the same tensors.

Readings taken where the workload descriptions leave a choice open:
* "Gaussian clusters (unit-norm centres, sigma s) plus N(0, n) noise" is read
  per element: key = centre + s * xi + n * zeta, xi, zeta ~ N(0, I).  Which
  cluster a token belongs to changes in runs (a new run starts at each token
  with probability 1/32), like topics in a document.
* Decode queries for clustered caches aim at one random cluster centre:
  q_h = sqrt(D) * centre + eps, eps ~ N(0, I), the cluster drawn per
  (sequence, KV head, step).  Values are N(0, 1) throughout.
* Needle blocks (MoBA-style workload): per KV head one unit direction u; keys
  in a needle block are N(0, I) + sqrt(D) * u and the group's queries are
  sqrt(D) * u + N(0, I).
* Semantic workload: the planted clusters are the blocks.  Keys are
  normalise(centre + 0.05 * xi); block sizes are log-normal (sigma 0.5)
  rescaled to sum to the context; positions are assigned to blocks by a
  random shuffle.  The store is built here from the planted assignment; the
  library's spherical k-means (bsa_build_semantic_index), started from the
  first key of each planted cluster, recovers exactly that assignment, so
  bsa_gather_rows over its order gives the same block-ordered store.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

CENTROID, CENTROID_NORM, MINMAX = 0, 1, 2


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    Hkv: int
    Hq: int
    D: int
    kv_dtype: torch.dtype
    L: int                      # tokens in the cache when decoding starts
    kind: int                   # summary kind
    block_size: int             # fixed block/page size; 0 = variable (semantic)
    topk: int                   # blocks; -1 = use budget_tokens
    budget_tokens: int
    sink: int
    window: int
    keep_current: bool
    refresh: int                # select every `refresh` decode steps
    steps: int                  # decode steps
    seed: int = 0
    n_clusters: int = 0
    cluster_sigma: float = 0.3
    noise_sigma: float = 0.1
    n_needles: int = 0          # tiny: needle keys; moba: needle blocks per KV head
    n_blocks: int = 0           # semantic: number of blocks
    chunk: int = 4096           # semantic prefill chunk / local part
    dense_below: int = 16384    # semantic: dense prefill while the prefix is shorter
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def L_max(self) -> int:
        """Rows each (batch, KV head) segment of the cache holds."""
        if self.block_size == 0:
            return self.L + self.chunk + self.steps + 64
        S = self.block_size
        return ((self.L + self.steps + S - 1) // S) * S + S

    def scaled(self, **kw) -> "Config":
        return replace(self, **kw)


def tiny(seed: int = 0) -> Config:
    """Batch 1, 1 KV head, 4 query heads, D 64, fp32; 4096 N(0,1) keys/values
    with 4 needle keys 3 q/|q|; blocks of 64, mean-pooled centroids, top-8,
    sink 64, window 128, one decode query."""
    return Config("tiny", 1, 1, 4, 64, torch.float32, 4096, CENTROID, 64, 8, 0, 64, 128,
                  False, 1, 1, seed, n_needles=4)


def quest(seed: int = 0) -> Config:
    """Quest-style paged decode: batch 4, 8 KV / 32 query heads, D 128, bf16;
    65,536-token cache of 64 Gaussian clusters (sigma 0.3) + N(0, 0.1) noise;
    pages of 16 with min/max bounds; budget 4096 tokens; sink 256; window
    1024; selection refreshed every 32 steps; 128 decode steps."""
    return Config("quest", 4, 8, 32, 128, torch.bfloat16, 65536, MINMAX, 16, -1, 4096, 256,
                  1024, False, 32, 128, seed, n_clusters=64)


def moba(seed: int = 0) -> Config:
    """MoBA-style block decode: batch 1, 8 KV / 64 query heads, D 128, bf16;
    131,072 N(0,1) keys with 16 needle blocks per KV head; blocks of 512,
    mean-pooled centroids, top-16, current block attended causally; 64 steps."""
    return Config("moba", 1, 8, 64, 128, torch.bfloat16, 131072, CENTROID, 512, 16, 0, 0, 0,
                  True, 1, 64, seed, n_needles=16)


def semantic(seed: int = 0) -> Config:
    """Semantic blocks: batch 1, 8 KV / 32 query heads, D 128, bf16; 524,288
    L2-normalised keys in 256 variable-size blocks (log-normal sizes, mean
    2048); K/V stored in block order; budget L/16; prefill in 4096-query
    chunks, dense while the prefix is under 16k; 32 decode steps."""
    return Config("semantic", 1, 8, 32, 128, torch.bfloat16, 524288, CENTROID_NORM, 0, -1,
                  524288 // 16, 0, 0, False, 1, 32, seed, n_blocks=256)


def largebatch(seed: int = 0) -> Config:
    """Large-batch decode: batch 64, 32 query / 8 KV heads, D 128, bf16;
    32,768 tokens of 32 clusters per sequence; pages of 32 with min/max;
    budget 8192; sink 256; window 512; selection every step; 256 steps."""
    return Config("largebatch", 64, 8, 32, 128, torch.bfloat16, 32768, MINMAX, 32, -1, 8192,
                  256, 512, False, 1, 256, seed, n_clusters=32)


def msa(seed: int = 0) -> Config:
    """MSA-shaped block decode (Attention mechanisms, MSA: blocks of 128,
    top-16 per GQA group = 2,048 tokens, the local block always kept):
    batch 2, 8 KV / 32 query heads, D 128, bf16; 131,072-token cache of 64
    Gaussian clusters (as quest); mean-pooled block keys; selection every
    step; 64 decode steps."""
    return Config("msa", 2, 8, 32, 128, torch.bfloat16, 131072, CENTROID, 128, 16, 0, 0, 0,
                  True, 1, 64, seed, n_clusters=64)


def quest_fp8(seed: int = 0) -> Config:
    """The Quest-style paged decode with the cache in FP8 (E4M3; Attention
    mechanisms, basic maths and the real cost: FP8 among the cache formats):
    batch 4, 8 KV / 32 query heads, D 128; 65,536-token cache of 64 Gaussian
    clusters; pages of 16 with min/max bounds; budget 4096 tokens; sink 256;
    window 1024; selection refreshed every 32 steps; 128 decode steps."""
    return replace(quest(seed), name="quest_fp8", kv_dtype=torch.float8_e4m3fn)


def largebatch_fp8(seed: int = 0) -> Config:
    """The large-batch decode with the cache in FP8 (E4M3): batch 64, 32 query
    / 8 KV heads, D 128; 32,768 tokens of 32 clusters per sequence; pages of
    32 with min/max; budget 8192; sink 256; window 512; selection every
    step; 256 steps."""
    return replace(largebatch(seed), name="largebatch_fp8", kv_dtype=torch.float8_e4m3fn)


CONFIGS = {"tiny": tiny, "quest": quest, "moba": moba, "semantic": semantic,
           "largebatch": largebatch, "msa": msa, "quest_fp8": quest_fp8,
           "largebatch_fp8": largebatch_fp8}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def _cluster_runs(g, n: int, n_clusters: int, device) -> torch.Tensor:
    """Cluster id per token, constant over runs that restart w.p. 1/32."""
    starts = torch.rand(n, generator=g, device=device) < (1.0 / 32.0)
    run = torch.cumsum(starts.to(torch.int64), 0)
    ids = torch.randint(0, n_clusters, (int(run[-1].item()) + 1,), generator=g, device=device)
    return ids[run]


class Workload:
    """Device-resident state of one config: cache, lengths and step inputs."""

    def __init__(self, cfg: Config, device="cpu"):
        self.cfg = cfg
        self.device = torch.device(device)
        g = _gen(self.device, cfg.seed)
        if cfg.block_size == 0:
            self._init_semantic(g)
        else:
            self._init_fixed(g)

    # ---------------------------------------------------------------- fixed
    def _init_fixed(self, g):
        c, dev = self.cfg, self.device
        B, H, D, Lm = c.B, c.Hkv, c.D, c.L_max
        self.K = torch.zeros(B, H, Lm, D, dtype=c.kv_dtype, device=dev)
        self.V = torch.zeros(B, H, Lm, D, dtype=c.kv_dtype, device=dev)
        self.cur_len = torch.full((B,), c.L, dtype=torch.int32, device=dev)
        if c.n_clusters:
            self.centres = _unit(torch.randn(B, H, c.n_clusters, D, generator=g, device=dev))
        if c.name == "moba":
            self.needle_dir = _unit(torch.randn(B, H, D, generator=g, device=dev))
        for b in range(B):
            for h in range(H):
                if c.n_clusters:
                    ids = _cluster_runs(g, c.L, c.n_clusters, dev)
                    k = (self.centres[b, h][ids]
                         + c.cluster_sigma * torch.randn(c.L, D, generator=g, device=dev)
                         + c.noise_sigma * torch.randn(c.L, D, generator=g, device=dev))
                else:
                    k = torch.randn(c.L, D, generator=g, device=dev)
                self.K[b, h, :c.L] = k.to(c.kv_dtype)
                self.V[b, h, :c.L] = torch.randn(c.L, D, generator=g, device=dev).to(c.kv_dtype)
        if c.name == "tiny":
            # one decode query; 4 needle keys 3 q0/|q0| at random positions
            self.q0 = torch.randn(B, c.Hq, D, generator=g, device=dev)
            pos = torch.randperm(c.L, generator=g, device=dev)[: c.n_needles]
            needle = 3.0 * _unit(self.q0[0, 0])
            self.K[0, 0, pos] = needle.to(c.kv_dtype)
            self.needle_pos = pos
        elif c.name == "moba":
            # needle blocks among the complete blocks before the current one
            S = c.block_size
            nb = max(c.L // S - 1, 0)
            n_need = min(c.n_needles, nb)
            self.needle_blocks = torch.stack([
                torch.randperm(max(nb, 1), generator=g, device=dev)[:n_need] for _ in range(B * H)
            ]).view(B, H, n_need)
            for b in range(B):
                for h in range(H):
                    add = (math.sqrt(D) * self.needle_dir[b, h]).to(torch.float32)
                    for j in self.needle_blocks[b, h].tolist():
                        blk = self.K[b, h, j * S:(j + 1) * S].float() + add
                        self.K[b, h, j * S:(j + 1) * S] = blk.to(c.kv_dtype)

    # ------------------------------------------------------------- semantic
    def _init_semantic(self, g):
        c, dev = self.cfg, self.device
        B, H, D, L, nb = c.B, c.Hkv, c.D, c.L, c.n_blocks
        Lm = c.L_max
        self.centres = _unit(torch.randn(B, H, nb, D, generator=g, device=dev))
        self.Kpos = torch.zeros(B, H, L + c.steps + 1, D, dtype=c.kv_dtype, device=dev)
        self.Vpos = torch.zeros_like(self.Kpos)
        self.labels = torch.zeros(B, H, L, dtype=torch.int64, device=dev)
        self.K = torch.zeros(B, H, Lm, D, dtype=c.kv_dtype, device=dev)
        self.V = torch.zeros_like(self.K)
        self.kv_pos = torch.full((B, H, Lm), -1, dtype=torch.int32, device=dev)
        self.block_offsets = torch.zeros(B, H, nb + 1, dtype=torch.int32, device=dev)
        for b in range(B):
            for h in range(H):
                w = torch.exp(0.5 * torch.randn(nb, generator=g, device=dev, dtype=torch.float64))
                n = torch.clamp(torch.floor(w / w.sum() * L), min=1).to(torch.int64)
                n[torch.argmax(n)] += L - int(n.sum().item())
                lab = torch.repeat_interleave(torch.arange(nb, device=dev), n)
                lab = lab[torch.randperm(L, generator=g, device=dev)]
                self.labels[b, h] = lab
                k = _unit(self.centres[b, h][lab] + 0.05 * torch.randn(L, D, generator=g, device=dev))
                v = torch.randn(L, D, generator=g, device=dev)
                self.Kpos[b, h, :L] = k.to(c.kv_dtype)
                self.Vpos[b, h, :L] = v.to(c.kv_dtype)
                order = torch.argsort(lab, stable=True)
                self.K[b, h, :L] = self.Kpos[b, h, order]
                self.V[b, h, :L] = self.Vpos[b, h, order]
                self.kv_pos[b, h, :L] = order.to(torch.int32)
                self.block_offsets[b, h, 1:] = torch.cumsum(n, 0).to(torch.int32)
                # local part for decode: the last `chunk` positions in position
                # order, stored after the blocks
                loc = torch.arange(L - c.chunk, L, device=dev)
                self.K[b, h, L:L + c.chunk] = self.Kpos[b, h, loc]
                self.V[b, h, L:L + c.chunk] = self.Vpos[b, h, loc]
                self.kv_pos[b, h, L:L + c.chunk] = loc.to(torch.int32)
        self.local_start = L                    # first row of the local part
        self.cur_len = torch.full((B,), L + c.chunk, dtype=torch.int32, device=dev)

    # ---------------------------------------------------------------- paged
    def paged(self, page_rows: int, spare_pages: int = 0, seed_offset: int = 7_000_001):
        """The cache laid out as a page pool ("Sparse long-context inference
        with self-indexing attention": the KV cache held as fixed-size pages):
        every sequence's rows cut into pages of `page_rows`, the pages placed
        at seeded random slots of a pool with `spare_pages` unused slots.
        Returns (K_pool, V_pool [n_pages, Hkv, page_rows, D], page_table int32
        [B, pages_per_seq]); logical page i of sequence b is pool page
        page_table[b, i]."""
        c, dev = self.cfg, self.device
        B, H, Lm, D = self.K.shape
        pps = -(-Lm // page_rows)
        n_pages = B * pps + spare_pages
        g = _gen(dev, c.seed + seed_offset)
        slots = torch.randperm(n_pages, generator=g, device=dev)[: B * pps]
        table = slots.view(B, pps).to(torch.int32).contiguous()
        Kp = torch.zeros(n_pages, H, page_rows, D, dtype=self.K.dtype, device=dev)
        Vp = torch.zeros_like(Kp)
        for b in range(B):
            for i in range(pps):
                r0, r1 = i * page_rows, min((i + 1) * page_rows, Lm)
                Kp[table[b, i], :, : r1 - r0] = self.K[b, :, r0:r1]
                Vp[table[b, i], :, : r1 - r0] = self.V[b, :, r0:r1]
        return Kp, Vp, table

    # --------------------------------------------------------------- inputs
    def decode_query(self, step: int) -> torch.Tensor:
        """Step `step`'s queries [B, Hq, D] fp32."""
        c, dev = self.cfg, self.device
        if c.name == "tiny":
            return self.q0.clone()
        g = _gen(dev, c.seed + 1 + step)
        eps = torch.randn(c.B, c.Hq, c.D, generator=g, device=dev)
        if c.name == "moba":
            aim = self.needle_dir
        else:
            n_c = self.centres.shape[2]
            pick = torch.randint(0, n_c, (c.B, c.Hkv), generator=g, device=dev)
            aim = torch.gather(self.centres, 2,
                               pick[:, :, None, None].expand(c.B, c.Hkv, 1, c.D))[:, :, 0]
        aim = aim.repeat_interleave(c.G, dim=1)
        return (math.sqrt(c.D) * aim + eps).contiguous()

    def decode_new_kv(self, step: int):
        """Step `step`'s new token K, V [B, Hkv, D] in the cache dtype."""
        c, dev = self.cfg, self.device
        g = _gen(dev, c.seed + 1 + step)
        torch.randn(c.B, c.Hq, c.D, generator=g, device=dev)   # the query's draw
        if c.n_clusters:
            torch.randint(0, c.n_clusters, (c.B, c.Hkv), generator=g, device=dev)
        if c.block_size == 0:
            pick = torch.randint(0, c.n_blocks, (c.B, c.Hkv), generator=g, device=dev)
            cen = torch.gather(self.centres, 2,
                               pick[:, :, None, None].expand(c.B, c.Hkv, 1, c.D))[:, :, 0]
            k = _unit(cen + 0.05 * torch.randn(c.B, c.Hkv, c.D, generator=g, device=dev))
        elif c.n_clusters:
            pick = torch.randint(0, c.n_clusters, (c.B, c.Hkv), generator=g, device=dev)
            cen = torch.gather(self.centres, 2,
                               pick[:, :, None, None].expand(c.B, c.Hkv, 1, c.D))[:, :, 0]
            k = (cen + c.cluster_sigma * torch.randn(c.B, c.Hkv, c.D, generator=g, device=dev)
                 + c.noise_sigma * torch.randn(c.B, c.Hkv, c.D, generator=g, device=dev))
        else:
            k = torch.randn(c.B, c.Hkv, c.D, generator=g, device=dev)
        v = torch.randn(c.B, c.Hkv, c.D, generator=g, device=dev)
        return k.to(c.kv_dtype).contiguous(), v.to(c.kv_dtype).contiguous()

    def prefill_queries(self, p: int, n: int) -> torch.Tensor:
        """Queries of positions [p, p+n) [n, Hq, D] bf16 (semantic workload):
        q = sqrt(D) * centre + N(0, I), the centre of a random block."""
        c, dev = self.cfg, self.device
        g = _gen(dev, c.seed + 1_000_003 + p)
        pick = torch.randint(0, c.n_blocks, (n, c.Hkv), generator=g, device=dev)
        cen = self.centres[0][torch.arange(c.Hkv, device=dev)[None, :], pick]   # [n, Hkv, D]
        q = math.sqrt(c.D) * cen.repeat_interleave(c.G, dim=1)
        q = q + torch.randn(n, c.Hq, c.D, generator=g, device=dev)
        return q.to(torch.bfloat16).contiguous()
