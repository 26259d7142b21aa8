"""Seeded synthetic inputs for the sparse-attention hot path.

This module only draws random tensors with the shapes, dtypes and value
distributions of the five workloads below.  It holds none of the method's
arithmetic: the CUDA library and the fp64 oracle both read what it makes,
and neither imports the other.

Workloads (seed = 1000 + workload number):

1 ``tiny``    decode, 1 sequence, L=2048.  Indexer H^I=4, d^I=64, integer q^I and
              k^I in [-4,4] stored as fp32, w from {0.25,0.5,1,2}; top-k 128.
              MLA 16 heads, d_c=512, d_R=64, N(0,1) bf16.
2 ``long``    decode, 32 sequences of L=32768.  Indexer H^I=64, d^I=128, integer
              q^I and k^I in [-8,8] stored as fp8 e4m3 (exact), w = 2^U{-4..1};
              top-k 2048.  MLA 128 heads, d_c=512, d_R=64, N(0,1) bf16.
3 ``ragged``  decode, 64 sequences, L_b ~ U[8192,131072]; shapes as ``long``;
              both caches in 64-token pages behind one shuffled page table.
4 ``prefill`` 4096 causal queries appended to a 61440-token history (L=65536);
              shapes as ``long``; query i sits at position 61440+i.
5 ``block``   block-sparse decode, 8 sequences of L=131072, 32 MHA heads,
              head_dim 128, N(0,1) bf16 Q/K/V; 64-token blocks, top-16 blocks,
              one sink block, a 512-token window.

Integer indexer inputs with power-of-two weights make every index score an
exact fp32 value, so both sides must produce identical Top-K sets.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch

PAGE = 64


@dataclass(frozen=True)
class DSAConfig:
    """Shapes and value recipe of one indexer -> Top-K -> sparse-MLA workload."""
    name: str
    seed: int
    n_seqs: int
    lens: tuple                 # history length per sequence (tokens in the cache)
    rows: int                   # query rows (decode: one per sequence)
    prefill_start: int = -1     # >=0: row i is the causal query at position prefill_start+i of sequence 0
    H_I: int = 64
    d_I: int = 128
    idx_dtype: str = "e4m3"     # "f32" or "e4m3"
    int_lo: int = -8
    int_hi: int = 8
    w_values: tuple = tuple(2.0 ** e for e in range(-4, 2))
    topk: int = 2048
    H: int = 128
    d_c: int = 512
    d_R: int = 64
    d_C: int = 128              # content dim before absorption; sets the softmax scale
    paged: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_C + self.d_R)

    @property
    def pages_per_seq(self) -> int:
        return max((l + PAGE - 1) // PAGE for l in self.lens)

    @property
    def L_max(self) -> int:
        return self.pages_per_seq * PAGE

    def n_visible(self) -> np.ndarray:
        if self.prefill_start >= 0:
            return np.arange(self.rows, dtype=np.int64) + self.prefill_start + 1
        return np.asarray(self.lens, dtype=np.int64)

    def seq_of_row(self) -> Optional[np.ndarray]:
        if self.prefill_start >= 0:
            return np.zeros(self.rows, dtype=np.int64)
        return None


@dataclass(frozen=True)
class BlockConfig:
    """Shapes of the block-sparse (mean-pooled block keys) decode workload."""
    name: str
    seed: int
    B: int
    L: int
    H: int
    D: int = 128
    block: int = 64
    top_blocks: int = 16
    sink_blocks: int = 1
    window: int = 512

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def n_blocks(self) -> int:
        return self.L // self.block


@dataclass(frozen=True)
class NSAConfig:
    """Shapes of the NSA three-branch decode workload: one decode query per
    head, H query heads in GQA groups of H / H_kv sharing one KV head."""
    name: str
    seed: int
    B: int
    L: int
    H: int
    H_kv: int
    D: int = 128
    block: int = 64
    top_blocks: int = 16
    window: int = 512

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def n_blocks(self) -> int:
        return self.L // self.block

    @property
    def G(self) -> int:
        return self.H // self.H_kv


@dataclass(frozen=True)
class CSAConfig:
    """Shapes of the CSA workload: DSA over m-token compressed entries plus a
    window of raw entries, one decode query per sequence."""
    name: str
    seed: int
    n_seqs: int
    L: int                      # raw tokens per sequence
    m: int = 4                  # tokens per compressed entry
    c: int = 512                # entry width (keys = values)
    H: int = 128                # query heads of the core attention
    H_I: int = 64
    d_I: int = 128
    topk: int = 2048
    window: int = 128
    int_lo: int = -8
    int_hi: int = 8
    w_values: tuple = tuple(2.0 ** e for e in range(-4, 2))

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.c)

    @property
    def n_c(self) -> int:
        return self.L // self.m

    @property
    def idx_pages(self) -> int:       # indexer pool pages per sequence (compressed keys)
        return max(1, (self.n_c + PAGE - 1) // PAGE)

    @property
    def n_cap(self) -> int:           # latent positions before the window slots
        return self.idx_pages * PAGE

    @property
    def lat_pages(self) -> int:       # latent pool pages per sequence (compressed entries, then window slots)
        return (self.n_cap + self.window + PAGE - 1) // PAGE


def _ragged_lens(seed: int, n: int, lo: int, hi: int) -> tuple:
    rng = np.random.Generator(np.random.PCG64(seed))
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=n))


TINY = DSAConfig(name="tiny", seed=1001, n_seqs=1, lens=(2048,), rows=1, H_I=4, d_I=64,
                 idx_dtype="f32", int_lo=-4, int_hi=4, w_values=(0.25, 0.5, 1.0, 2.0),
                 topk=128, H=16)
LONG = DSAConfig(name="long", seed=1002, n_seqs=32, lens=(32768,) * 32, rows=32)
RAGGED = DSAConfig(name="ragged", seed=1003, n_seqs=64,
                   lens=_ragged_lens(1003, 64, 8192, 131072), rows=64, paged=True)
PREFILL = DSAConfig(name="prefill", seed=1004, n_seqs=1, lens=(65536,), rows=4096,
                    prefill_start=61440)
BLOCK = BlockConfig(name="block", seed=1005, B=8, L=131072, H=32)

NSA = NSAConfig(name="nsa", seed=1006, B=8, L=131072, H=32, H_kv=4)

DSA_CONFIGS = {c.name: c for c in (TINY, LONG, RAGGED, PREFILL)}
BLOCK_CONFIGS = {BLOCK.name: BLOCK}
NSA_CONFIGS = {NSA.name: NSA}
CSA = CSAConfig(name="csa", seed=1007, n_seqs=32, L=131072)
CSA_CONFIGS = {CSA.name: CSA}


def small_dsa(base: DSAConfig, **kw) -> DSAConfig:
    """A copy of ``base`` with some fields replaced (test-sized variants)."""
    return replace(base, **kw)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _ints(g, shape, lo, hi, device) -> torch.Tensor:
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.int32).to(torch.float32)


def _normal_bf16(g, shape, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def page_layout(cfg: DSAConfig, seed: int):
    """Physical page ids for every (sequence, logical page).

    Paged: every sequence owns ceil(L_b/64) pages drawn from a seeded
    permutation of the pool; unused table entries are -1.
    Contiguous: no table; sequence b's logical page p is physical page
    b*pages_per_seq + p.
    Returns (page_table or None, number of pages in the pool).
    """
    pps = cfg.pages_per_seq
    if not cfg.paged:
        return None, cfg.n_seqs * pps
    need = [(l + PAGE - 1) // PAGE for l in cfg.lens]
    total = int(sum(need))
    rng = np.random.Generator(np.random.PCG64(seed + 77))
    perm = rng.permutation(total).astype(np.int32)
    table = np.full((cfg.n_seqs, pps), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, total


def dsa_inputs(cfg: DSAConfig, device="cpu", seed: Optional[int] = None) -> dict:
    """Draw every tensor of one indexer -> Top-K -> sparse-MLA step.

    Returns a dict of torch tensors on ``device`` plus the host-side metadata:
      q_idx [rows,H_I,d_I] (fp32 or fp8 e4m3), w [rows,H_I] fp32,
      k_idx_cache [pages*64, d_I] (pool of 64-token pages),
      q_lat [rows,H,d_c] bf16, q_rope [rows,H,d_R] bf16,
      c_cache [pages*64, d_c] bf16, kr_cache [pages*64, d_R] bf16,
      page_table [n_seqs, pages_per_seq] int32 or None, seq_lens [n_seqs] int32,
      n_visible [rows] int32, seq_of_row [rows] int32 or None.
    """
    seed = cfg.seed if seed is None else seed
    dev = torch.device(device)
    g = _gen(dev, seed)
    table, n_pages = page_layout(cfg, seed)
    pool_rows = n_pages * PAGE
    q_idx = _ints(g, (cfg.rows, cfg.H_I, cfg.d_I), cfg.int_lo, cfg.int_hi, dev)
    k_idx = _ints(g, (pool_rows, cfg.d_I), cfg.int_lo, cfg.int_hi, dev)
    if cfg.idx_dtype == "e4m3":
        q_idx = q_idx.to(torch.float8_e4m3fn)
        k_idx = k_idx.to(torch.float8_e4m3fn)
    wv = torch.tensor(cfg.w_values, dtype=torch.float32, device=dev)
    w = wv[torch.randint(0, len(cfg.w_values), (cfg.rows, cfg.H_I), generator=g, device=dev)]
    q_lat = _normal_bf16(g, (cfg.rows, cfg.H, cfg.d_c), dev)
    q_rope = _normal_bf16(g, (cfg.rows, cfg.H, cfg.d_R), dev)
    c_cache = _normal_bf16(g, (pool_rows, cfg.d_c), dev)
    kr_cache = _normal_bf16(g, (pool_rows, cfg.d_R), dev)
    out = dict(
        cfg=cfg, q_idx=q_idx, w=w.contiguous(), k_idx_cache=k_idx, q_lat=q_lat, q_rope=q_rope,
        c_cache=c_cache, kr_cache=kr_cache,
        page_table=None if table is None else torch.from_numpy(table).to(dev),
        seq_lens=torch.tensor(cfg.lens, dtype=torch.int32, device=dev),
        n_visible=torch.from_numpy(cfg.n_visible().astype(np.int32)).to(dev),
        seq_of_row=None if cfg.seq_of_row() is None else torch.from_numpy(cfg.seq_of_row().astype(np.int32)).to(dev),
    )
    return out


def physical_rows(cfg: DSAConfig, page_table: Optional[np.ndarray], seq: int, positions: np.ndarray) -> np.ndarray:
    """Pool row of each logical position of sequence ``seq`` (plain page lookup)."""
    positions = np.asarray(positions, dtype=np.int64)
    page = positions // PAGE
    if page_table is None:
        phys = seq * cfg.pages_per_seq + page
    else:
        phys = np.asarray(page_table)[seq, page].astype(np.int64)
    return phys * PAGE + positions % PAGE


def block_inputs(cfg: BlockConfig, device="cpu", seed: Optional[int] = None) -> dict:
    """Draw q [B,H,D], K and V [B,L,H,D] (all N(0,1) bf16) for the block-sparse step."""
    seed = cfg.seed if seed is None else seed
    dev = torch.device(device)
    g = _gen(dev, seed)
    q = _normal_bf16(g, (cfg.B, cfg.H, cfg.D), dev)
    K = _normal_bf16(g, (cfg.B, cfg.L, cfg.H, cfg.D), dev)
    V = _normal_bf16(g, (cfg.B, cfg.L, cfg.H, cfg.D), dev)
    return dict(cfg=cfg, q=q, K=K, V=V)


def csa_inputs(cfg: CSAConfig, device="cpu", seed: Optional[int] = None) -> dict:
    """Draw every input of the CSA step.

    Entry streams (the two per-token projections the compression merges) and
    their compression weights, [n_seqs, L, width] bf16, N(0,1): Ca, Cb, Za, Zb
    (width c) and the indexer-key streams CIa, CIb, ZIa, ZIb (width d_I);
    position biases Ba, Bb [m, c], BIa, BIb [m, d_I] fp32.  The indexer-key
    entry streams are integers in [int_lo, int_hi] that repeat over the 2m rows
    each compressed entry merges (group g of stream a and group g-1 of stream
    b carry the same integers), so every compressed indexer key is that
    integer vector exactly and the index scores are exact in fp32.
    Query side: q_idx [n_seqs, H_I, d_I] e4m3 integers, w powers of two, q
    [n_seqs, H, c] bf16, q_rope zeros [n_seqs, H, 64].
    Caches the compression fills: idx_pool [n_seqs * idx_pages * 64, d_I] e4m3
    and lat_pool [n_seqs * lat_pages * 64, c] bf16, whose window slots
    (latent positions n_cap .. n_cap + window - 1 of each sequence) hold the
    raw entries Ca of the last `window` tokens, oldest first."""
    seed = cfg.seed if seed is None else seed
    dev = torch.device(device)
    g = _gen(dev, seed)
    S, L, m, c, dI = cfg.n_seqs, cfg.L, cfg.m, cfg.c, cfg.d_I
    Ca, Cb, Za, Zb = (_normal_bf16(g, (S, L, c), dev) for _ in range(4))
    Ba, Bb = (torch.randn((m, c), generator=g, device=dev) for _ in range(2))
    n_groups = (L + m - 1) // m
    V = _ints(g, (S, n_groups + 1, dI), cfg.int_lo, cfg.int_hi, dev)
    CIa = V[:, :n_groups].repeat_interleave(m, dim=1)[:, :L].to(torch.bfloat16).contiguous()
    CIb = V[:, 1:n_groups + 1].repeat_interleave(m, dim=1)[:, :L].to(torch.bfloat16).contiguous()
    ZIa, ZIb = (_normal_bf16(g, (S, L, dI), dev) for _ in range(2))
    BIa, BIb = (torch.randn((m, dI), generator=g, device=dev) for _ in range(2))
    q_idx = _ints(g, (S, cfg.H_I, dI), cfg.int_lo, cfg.int_hi, dev).to(torch.float8_e4m3fn)
    wv = torch.tensor(cfg.w_values, dtype=torch.float32, device=dev)
    w = wv[torch.randint(0, len(cfg.w_values), (S, cfg.H_I), generator=g, device=dev)].contiguous()
    q = _normal_bf16(g, (S, cfg.H, c), dev)
    q_rope = torch.zeros((S, cfg.H, 64), dtype=torch.bfloat16, device=dev)
    idx_pool = torch.zeros((S * cfg.idx_pages * PAGE, dI), dtype=torch.float8_e4m3fn, device=dev)
    lat_pool = torch.zeros((S * cfg.lat_pages * PAGE, c), dtype=torch.bfloat16, device=dev)
    wl = min(cfg.window, L)
    lat3 = lat_pool.view(S, cfg.lat_pages * PAGE, c)
    lat3[:, cfg.n_cap: cfg.n_cap + wl] = Ca[:, L - wl:]
    return dict(cfg=cfg, Ca=Ca, Cb=Cb, Za=Za, Zb=Zb, Ba=Ba, Bb=Bb, CIa=CIa, CIb=CIb, ZIa=ZIa, ZIb=ZIb, BIa=BIa,
                BIb=BIb, q_idx=q_idx, w=w, q=q, q_rope=q_rope, idx_pool=idx_pool, lat_pool=lat_pool,
                n_visible=torch.full((S,), cfg.n_c, dtype=torch.int32, device=dev),
                seq_lens=torch.full((S,), L, dtype=torch.int32, device=dev))


def nsa_inputs(cfg: NSAConfig, device="cpu", seed: Optional[int] = None) -> dict:
    """Draw q [B,H,D], K and V [B,L,H_kv,D] (all N(0,1) bf16) and the branch
    gates [B,H,3] (fp32, uniform in (0,1): values a sigmoid can take)."""
    seed = cfg.seed if seed is None else seed
    dev = torch.device(device)
    g = _gen(dev, seed)
    q = _normal_bf16(g, (cfg.B, cfg.H, cfg.D), dev)
    K = _normal_bf16(g, (cfg.B, cfg.L, cfg.H_kv, cfg.D), dev)
    V = _normal_bf16(g, (cfg.B, cfg.L, cfg.H_kv, cfg.D), dev)
    gates = torch.rand((cfg.B, cfg.H, 3), generator=g, device=dev, dtype=torch.float32)
    return dict(cfg=cfg, q=q, K=K, V=V, gates=gates)
