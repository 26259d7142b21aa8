#!/usr/bin/env python
"""Benchmark of the sparse-attention hot path on B200.

One step = the whole decode path over one batch: lightning indexer ->
exact Top-K -> sparse MLA, i.e. one query per sequence of the workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config long|ragged|tiny|prefill|block|nsa|csa|crossover]
                    [--impl native|reference]

Default workload: long decode, 32 sequences x 32768 tokens, H^I=64 fp8
indexer, top-2048, 128-head sparse MLA (latent 512 + RoPE 64, bf16).  With N
GPUs (torchrun, one process per GPU) every rank runs its own batch of the
same shape (weak scaling, no data-path collective); the step time is the max
over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DECODE_METRIC = "sparse-MLA decode queries/s (indexer+topk+attn) at L=32K/128K; % HBM roofline"
L2_BYTES = 126 * 10**6  # B200 L2
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2

# dram__bytes_read.sum + dram__bytes_write.sum per launch of the roofline
# kernel of a workload, from one ncu capture, with the sha256 prefix of the
# kernel source it was taken on (the figure is reported only while they match).
TRAFFIC = {
    # mla_kernel only (the split combine's traffic is not in the figure)
    "long": {"kernel": "sparse_mla.cu", "stage": "attn", "bytes_per_launch": 83477760, "src_sha": "0b24f374f08045e9"},
    # captured on the first 16 sequences, scaled by the key bytes to the full launch (x 3.955)
    "ragged": {"kernel": "index_scores.cu", "stage": "indexer", "bytes_per_launch": 592467514,
               "src_sha": "82268133da2ff55d"},
    # block_sparse_cluster_kernel<1> on the full block workload (one pass: no scaling)
    "block": {"kernel": "block_sparse.cu", "bytes_per_launch": 483272448, "src_sha": "e02282be07fa6780"},
    "nsa": {"kernel": "nsa.cu", "bytes_per_launch": 59074304, "src_sha": "e49c849dfa2ed8a1"},
}


def src_sha(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# ---------------------------------------------------------------- work model
def decode_bytes(cfg: W.DSAConfig):
    """Algorithmic bytes of one decode step: every visible indexer key once plus
    every selected latent row (512 bf16 + 64 bf16 RoPE key) once."""
    esize = 1 if cfg.idx_dtype == "e4m3" else 4
    nv = cfg.n_visible()
    keys = int(nv.sum()) * cfg.d_I * esize
    rows = int(np.minimum(nv, cfg.topk).sum()) * (cfg.d_c + cfg.d_R) * 2
    return keys, rows


def prefill_flops(cfg: W.DSAConfig):
    nv = cfg.n_visible().astype(np.float64)
    idx = float((nv * 2 * cfg.H_I * cfg.d_I).sum())
    mla = float((np.minimum(nv, cfg.topk) * cfg.H * 2 * (cfg.d_c + cfg.d_R + cfg.d_c)).sum())
    return idx, mla


def step_working_set(cfg, step) -> int:
    """Distinct bytes one step reads (its working set for L2 purposes)."""
    if isinstance(cfg, W.DSAConfig):
        if cfg.prefill_start >= 0:  # every query row of the chunk reads the same history
            esize = 1 if cfg.idx_dtype == "e4m3" else 4
            return int(cfg.n_seqs * cfg.L_max * (cfg.d_I * esize + (cfg.d_c + cfg.d_R) * 2))
        return int(sum(decode_bytes(cfg)))
    if isinstance(cfg, W.CSAConfig):
        return int(sum(csa_bytes(cfg)))
    if isinstance(cfg, W.NSAConfig):
        return int(nsa_bytes(cfg))
    return int(block_bytes(cfg, step.union_tokens)[0])


def block_union_tokens(cfg: W.BlockConfig, sel: np.ndarray) -> int:
    """Tokens attended over all (sequence, head) pairs: the union of the
    chosen blocks (sel [B, H, top], -1 padded), the sink blocks and the
    window, each token counted once per pair."""
    total = 0
    w0 = max(0, cfg.L - cfg.window)
    for b in range(sel.shape[0]):
        for h in range(sel.shape[1]):
            m = np.zeros(cfg.L, dtype=bool)
            m[w0:] = True
            m[: min(cfg.L, cfg.sink_blocks * cfg.block)] = True
            for n in sel[b, h]:
                if n >= 0:
                    m[n * cfg.block:(n + 1) * cfg.block] = True
            total += int(m.sum())
    return total


def block_bytes(cfg: W.BlockConfig, union_tokens: int):
    """Algorithmic bytes of one block-sparse decode step: for every (sequence,
    head) the pooled keys of every complete block (fp32), the K and V rows of
    the attended union (bf16), the query and the output; `union_tokens` is
    the union size summed over the pairs.  Returns (bytes, union_tokens)."""
    pairs = cfg.B * cfg.H
    pooled = pairs * cfg.n_blocks * cfg.D * 4
    kv = union_tokens * 2 * cfg.D * 2
    qo = pairs * cfg.D * (2 + 4)
    return pooled + kv + qo, union_tokens


def nsa_bytes(cfg: W.NSAConfig):
    """Algorithmic bytes of one NSA decode step, every (sequence, KV head):
    the compressed K and V rows of every complete block, the K and V rows of
    the selected blocks and of the window, the group's queries, gates and
    outputs."""
    nb = cfg.n_blocks
    per_group = (2 * nb * cfg.D * 2 + min(cfg.top_blocks, nb) * cfg.block * 2 * cfg.D * 2
                 + min(cfg.window, cfg.L) * 2 * cfg.D * 2 + cfg.G * (cfg.D * 2 + 12 + cfg.D * 4))
    return per_group * cfg.B * cfg.H_kv


def csa_bytes(cfg: W.CSAConfig):
    """Algorithmic bytes of one CSA decode step: every compressed indexer key
    once (e4m3, d_I bytes), then every selected entry and window slot once
    (a 512-wide bf16 latent row plus the 64 dims the attention kernel reads
    as its RoPE key), per sequence."""
    keys = cfg.n_seqs * cfg.n_c * cfg.d_I
    rows = cfg.n_seqs * (min(cfg.topk, cfg.n_c) + min(cfg.window, cfg.L)) * (cfg.c + 64) * 2
    return keys, rows


# ---------------------------------------------------------------- ranks
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(values, world_size: int, device):
    """Element-wise max over ranks (identity for one rank)."""
    if world_size == 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def rank_seed(base: int, rank: int) -> int:
    return base + 7919 * rank


# ---------------------------------------------------------------- clocks
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- native arm
class DecodeStep:
    """Buffers and launches of one indexer -> Top-K -> sparse-MLA step."""

    def __init__(self, inp, sa, topk_path: str = "scores", out_dtype=torch.bfloat16):
        self.sa, self.inp, self.cfg = sa, inp, inp["cfg"]
        cfg, dev = self.cfg, inp["q_idx"].device
        self.idx = torch.empty(cfg.rows, cfg.topk, dtype=torch.int32, device=dev)
        # the attention output as the up-projection reads it (bf16; fp32 accumulation)
        self.out = torch.empty(cfg.rows, cfg.H, cfg.d_c, dtype=out_dtype, device=dev)
        self.lse = torch.empty(cfg.rows, cfg.H, dtype=torch.float32, device=dev)
        self.prefill = cfg.prefill_start >= 0
        # decode with one query row per sequence on the tensor-core indexer:
        # the indexer keeps only the keys that can still be in the Top-K
        # (candidates) and the Top-K selects from them; otherwise the indexer
        # writes every score and counts each row's first Top-K digit, and the
        # Top-K starts from those counts.  Both leave their counts cleared.
        self.cand_path = (topk_path == "cand" and not self.prefill and inp["seq_of_row"] is None
                          and cfg.idx_dtype == "e4m3" and cfg.d_I == 128 and cfg.H_I in (16, 32, 64, 128))
        if self.cand_path:
            self.scores = None
            self.cand, self.cand_cnt, self.hist = sa.candidate_buffers(cfg.rows, cfg.pages_per_seq * 64, dev)
        else:
            self.scores = torch.empty(cfg.rows, cfg.L_max, dtype=torch.float32, device=dev)
            self.hist = sa.topk_histogram(cfg.rows, dev)
        size = sa.sparse_mla_prefill_workspace_size if self.prefill else sa.sparse_mla_workspace_size
        self.ws = torch.empty(size(cfg.rows, cfg.H, cfg.topk, cfg.d_c), dtype=torch.uint8, device=dev)
        # decode splits keys (and adds the combine launch) when its workspace holds partial states
        combine = not self.prefill and (sa.sparse_mla_workspace_size(cfg.rows, cfg.H, cfg.topk, cfg.d_c) >
                                        sa.sparse_mla_prefill_workspace_size(cfg.rows, cfg.H, cfg.topk, cfg.d_c))
        self.launches_per_step = 3 + (1 if combine else 0)

    def indexer(self):
        i, c = self.inp, self.cfg
        if self.cand_path:
            self.sa.index_candidates(i["q_idx"], i["w"], i["k_idx_cache"], i["n_visible"], c.pages_per_seq, c.topk,
                                     self.cand, self.cand_cnt, self.hist, page_table=i["page_table"])
        else:
            self.sa.index_scores(i["q_idx"], i["w"], i["k_idx_cache"], i["n_visible"], c.pages_per_seq,
                                 page_table=i["page_table"], seq_of_row=i["seq_of_row"], scores=self.scores,
                                 hist=self.hist)

    def rest(self):
        self.topk()
        self.attn()

    def topk(self):
        if self.cand_path:
            self.sa.topk_from_candidates(self.cand, self.cand_cnt, self.inp["n_visible"], self.cfg.topk, self.hist,
                                         idx_out=self.idx)
        else:
            self.sa.topk_select(self.scores, self.inp["n_visible"], self.cfg.topk, idx_out=self.idx,
                                hist=self.hist)

    def kept_candidates(self) -> int:
        """Candidates the indexer keeps over all rows in one step (0 on the
        score path); runs one indexer launch and one Top-K launch."""
        if not self.cand_path:
            return 0
        self.indexer()
        kept = int(self.cand_cnt.sum())
        self.topk()
        return kept

    def attn(self):
        i, c = self.inp, self.cfg
        if self.prefill:
            self.sa.sparse_mla_prefill(i["q_lat"], i["q_rope"], i["c_cache"], i["kr_cache"], self.idx, c.scale,
                                       c.pages_per_seq, page_table=i["page_table"], seq_of_row=i["seq_of_row"],
                                       out=self.out, lse=self.lse, workspace=self.ws)
        else:
            self.sa.sparse_mla_decode(i["q_lat"], i["q_rope"], i["c_cache"], i["kr_cache"], self.idx, c.scale,
                                      c.pages_per_seq, page_table=i["page_table"], seq_of_row=i["seq_of_row"],
                                      out=self.out, lse=self.lse, workspace=self.ws)


class BlockStep:
    def __init__(self, inp, sa):
        self.sa, self.inp, self.cfg = sa, inp, inp["cfg"]
        c = self.cfg
        self.pooled = sa.block_mean_pool(inp["K"], c.block)  # once, when the blocks completed
        self.out = torch.empty(c.B, c.H, c.D, dtype=torch.float32, device=inp["q"].device)
        self.launches_per_step = 1
        # the union each pair attends to (for the byte model), from one call outside the timing
        sel = torch.empty(c.B, c.H, c.top_blocks, dtype=torch.int32, device=inp["q"].device)
        sa.block_sparse_attn(inp["q"], self.pooled, inp["K"], inp["V"], c.block, c.top_blocks, c.sink_blocks,
                             c.window, c.scale, out=self.out, sel_blocks=sel)
        self.union_tokens = block_union_tokens(c, sel.cpu().numpy())

    def indexer(self):
        i, c = self.inp, self.cfg
        self.sa.block_sparse_attn(i["q"], self.pooled, i["K"], i["V"], c.block, c.top_blocks, c.sink_blocks,
                                  c.window, c.scale, out=self.out)

    def rest(self):
        pass

    def topk(self):
        pass

    def attn(self):
        pass


class NsaStep:
    def __init__(self, inp, sa):
        self.sa, self.inp, self.cfg = sa, inp, inp["cfg"]
        c = self.cfg
        self.Kc, self.Vc = sa.nsa_compress(inp["K"], inp["V"], c.block)  # once, when the blocks completed
        self.out = torch.empty(c.B, c.H, c.D, dtype=torch.float32, device=inp["q"].device)
        self.launches_per_step = 1

    def indexer(self):
        i, c = self.inp, self.cfg
        self.sa.nsa_decode(i["q"], i["K"], i["V"], self.Kc, self.Vc, i["gates"], c.block, c.top_blocks, c.window,
                           c.scale, out=self.out)

    def rest(self):
        pass

    def topk(self):
        pass

    def attn(self):
        pass


class CsaStep:
    """indexer over the compressed keys -> Top-K -> window slots + sparse
    attention over the selected entries and the window."""

    def __init__(self, inp, sa, out_dtype=torch.bfloat16):
        self.sa, self.inp, self.cfg = sa, inp, inp["cfg"]
        c, dev = self.cfg, inp["q"].device
        S = c.n_seqs
        lat = inp["lat_pool"].view(S, c.lat_pages * 64, c.c)
        idx = inp["idx_pool"].view(S, c.idx_pages * 64, c.d_I)
        self.compress = lambda: (  # noqa: E731  (run as groups complete; timed on its own)
            sa.csa_compress(inp["Ca"], inp["Cb"], inp["Za"], inp["Zb"], inp["Ba"], inp["Bb"], c.m, inp["lat_pool"],
                            lat.stride(0), lat.stride(1)),
            sa.csa_compress(inp["CIa"], inp["CIb"], inp["ZIa"], inp["ZIb"], inp["BIa"], inp["BIb"], c.m,
                            inp["idx_pool"], idx.stride(0), idx.stride(1)))
        self.compress()
        self.scores = torch.empty(S, c.idx_pages * 64, dtype=torch.float32, device=dev)
        self.hist = sa.topk_histogram(S, dev)
        self.idx = torch.empty(S, c.topk, dtype=torch.int32, device=dev)
        self.slots = torch.empty(S, c.topk + c.window, dtype=torch.int32, device=dev)
        self.out = torch.empty(S, c.H, c.c, dtype=out_dtype, device=dev)
        self.ws = torch.empty(max(1, sa.sparse_mla_workspace_size(S, c.H, c.topk + c.window, c.c)),
                              dtype=torch.uint8, device=dev)
        combine = sa.sparse_mla_workspace_size(S, c.H, c.topk + c.window, c.c) > \
            sa.sparse_mla_prefill_workspace_size(S, c.H, c.topk + c.window, c.c)
        self.launches_per_step = 4 + (1 if combine else 0)

    def indexer(self):
        i, c = self.inp, self.cfg
        self.sa.index_scores(i["q_idx"], i["w"], i["idx_pool"], i["n_visible"], c.idx_pages, scores=self.scores,
                             hist=self.hist)

    def rest(self):
        self.topk()
        self.attn()

    def topk(self):
        self.sa.topk_select(self.scores, self.inp["n_visible"], self.cfg.topk, idx_out=self.idx, hist=self.hist)

    def attn(self):
        i, c = self.inp, self.cfg
        self.sa.csa_window_index(self.idx, i["seq_lens"], c.window, c.n_cap, idx_out=self.slots)
        self.sa.sparse_mla_decode(i["q"], i["q_rope"], i["lat_pool"], i["lat_pool"], self.slots, c.scale,
                                  c.lat_pages, out=self.out, workspace=self.ws)


def time_compress(step, K: int, flush, hbm: float):
    """The CSA compression of the whole history (both entry kinds), timed on
    its own: in decode it runs once per m tokens, outside the step."""
    c = step.cfg
    for _ in range(2):
        step.compress()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        flush.zero_()
        a.record()
        step.compress()
        b.record()
    torch.cuda.synchronize()
    us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
    nbytes = c.n_seqs * c.L * 4 * 2 * (c.c + c.d_I) + c.n_seqs * c.n_c * (c.c * 2 + c.d_I)
    return {"kernel": "csa_compress_kernel x2", "us": round(us, 1), "tokens_per_s": round(c.n_seqs * c.L / (us * 1e-6), 1),
            "bytes": nbytes, "hbm_gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
            "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / hbm, 4)}


def capture_step(step):
    """One step (all its library launches) captured as a CUDA graph on a side
    stream, after the warm-up; None if a launch of the step cannot be captured."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.stream(s):
            step.indexer()
            step.rest()
            s.synchronize()
            with torch.cuda.graph(g, stream=s):
                step.indexer()
                step.rest()
    except RuntimeError:
        torch.cuda.synchronize()
        return None
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def time_graph(g, K: int, flush):
    """K replays of the step's graph, each bracketed by CUDA events on the
    launching stream (no event between the step's kernels); the L2 flush runs
    between replays outside the events.  Per-step times in ms."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for e in ev:
        flush.zero_()
        e[0].record()
        g.replay()
        e[1].record()
    torch.cuda.synchronize()
    return [e[0].elapsed_time(e[1]) for e in ev]


def time_steps(step, K: int, flush):
    """K steps, each bracketed by CUDA events on the launching stream (torch's
    current stream, which the library calls use); the L2 flush runs between
    steps outside the events.  Returns per-step times and the per-step times of
    the three stages (indexer, Top-K, attention) in ms."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    for e in ev:
        flush.zero_()
        e[0].record()
        step.indexer()
        e[1].record()
        step.topk()
        e[2].record()
        step.attn()
        e[3].record()
    torch.cuda.synchronize()
    return ([e[0].elapsed_time(e[3]) for e in ev],
            [[e[j].elapsed_time(e[j + 1]) for e in ev] for j in range(3)])


def time_projections(step, K: int, flush, hbm: float):
    """The per-head projections around sparse MLA (query absorption with U_K,
    up-projection with U_V), timed on their own with synthetic weights of the
    workload's shapes (d_C=128, d_v=128): outside the metric's step, which
    starts from the absorbed query and ends at the latent output."""
    import sparse_attention_07_b200 as sa
    cfg, dev = step.cfg, step.out.device
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed + 77)
    q_c = (torch.randn(cfg.rows, cfg.H, cfg.d_C, generator=g, device=dev)).to(torch.bfloat16)
    U_K = (torch.randn(cfg.H, cfg.d_C, cfg.d_c, generator=g, device=dev) / cfg.d_C ** 0.5).to(torch.bfloat16)
    U_V = (torch.randn(cfg.H, 128, cfg.d_c, generator=g, device=dev) / cfg.d_c ** 0.5).to(torch.bfloat16)
    q_lat = torch.empty(cfg.rows, cfg.H, cfg.d_c, dtype=torch.bfloat16, device=dev)
    out = torch.empty(cfg.rows, cfg.H, 128, dtype=torch.float32, device=dev)
    res = {}
    for name, fn, w in (("absorb", lambda: sa.mla_absorb_query(q_c, U_K, q_lat=q_lat), U_K),
                        ("up_project", lambda: sa.mla_up_project(step.out, U_V, out=out), U_V)):
        for _ in range(3):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for a, b in ev:
            flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
        nbytes = w.numel() * 2  # the weights are read once; the activations are a few hundred KB
        res[name] = {"kernel": "head_gemm_kernel", "us": round(us, 2), "weight_bytes": nbytes,
                     "hbm_gbs": round(nbytes / (us * 1e-6) / 1e9, 1), "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / hbm, 4)}
    return res


E2E_SLOTS = 3  # steps in flight in the end-to-end pipeline


def pack_layout(tensors):
    """(offset, bytes) of each tensor in one packed byte buffer (pieces start
    on 16-byte boundaries), and the buffer's size."""
    offs, total = [], 0
    for t in tensors:
        nb = t.numel() * t.element_size()
        offs.append((total, nb))
        total += (nb + 15) // 16 * 16
    return offs, total


def pack_host(tensors, offs, total):
    """The tensors' bytes at their offsets in one host uint8 buffer."""
    buf = torch.zeros(total, dtype=torch.uint8)
    for t, (o, nb) in zip(tensors, offs):
        buf[o:o + nb].copy_(t.detach().contiguous().view(-1).view(torch.uint8).cpu())
    return buf


def e2e_steps(step, K: int, flush, flush_each: bool):
    """The step through the public API as a serving loop runs it: every step's
    query inputs are copied in from pinned host memory (packed in one buffer,
    one transfer) and its output is read
    back to pinned host memory, on their own streams, so that the copies of
    neighbouring steps overlap the compute.  Per step, on the compute stream:
    the inputs move from the step's slot into the step's input tensors (a
    device copy), L2 is flushed when the step's working set would fit in it
    (`flush_each`), the step runs, and its output moves to the slot (a device
    copy) for the read-back.  A slot is reused only after its read-back
    finished.  One pair of events brackets all K steps (all copies, flushes
    and device copies inside); returns [per-step ms] * K."""
    inp = step.inp
    if isinstance(step, DecodeStep):
        names = ["q_idx", "w", "q_lat", "q_rope"]
    elif isinstance(step, CsaStep):
        names = ["q_idx", "w", "q", "q_rope"]
    elif isinstance(step, NsaStep):
        names = ["q", "gates"]
    else:
        names = ["q"]
    result = step.out
    # two slots when a step's output is large (the prefill chunk's is 1 GB)
    S = E2E_SLOTS if result.numel() * result.element_size() <= (256 << 20) else 2
    # the step's inputs packed in one pinned buffer: one host-to-device copy
    # per step, split into the step's tensors on the device
    offs, total = pack_layout([inp[n] for n in names])
    offs = dict(zip(names, offs))
    host_in = pack_host([inp[n] for n in names], offs.values(), total).pin_memory()
    host_out = [torch.empty(result.shape, dtype=result.dtype).pin_memory() for _ in range(S)]
    dev_in = [torch.empty(total, dtype=torch.uint8, device=result.device) for _ in range(S)]
    dev_out = [torch.empty_like(result) for _ in range(S)]
    h2d = sum(nb for _, nb in offs.values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(K)]
    comp_done = [torch.cuda.Event() for _ in range(K)]
    out_done = [torch.cuda.Event() for _ in range(K)]
    cur = torch.cuda.current_stream()
    for st in (s_in, s_comp, s_out):
        st.wait_stream(cur)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for st in (s_in, s_comp, s_out):
        st.wait_event(e0)
    for i in range(K):
        slot = i % S
        with torch.cuda.stream(s_in):
            if i >= S:
                s_in.wait_event(comp_done[i - S])  # the slot's inputs were taken
            dev_in[slot].copy_(host_in, non_blocking=True)
            in_done[i].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[i])
            if i >= S:
                s_comp.wait_event(out_done[i - S])  # the slot's output was read back
            for n in names:
                o, nb = offs[n]
                inp[n].view(-1).view(torch.uint8).copy_(dev_in[slot][o:o + nb], non_blocking=True)
            if flush_each:
                flush.zero_()
            step.indexer()
            step.rest()
            dev_out[slot].copy_(result, non_blocking=True)
            comp_done[i].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[i])
            host_out[slot].copy_(dev_out[slot], non_blocking=True)
            out_done[i].record(s_out)
    for st in (s_in, s_comp, s_out):
        cur.wait_stream(st)
    e1.record(cur)
    torch.cuda.synchronize()
    per = e0.elapsed_time(e1) / K
    return [per] * K, h2d, d2h


def cpu_baseline(inp, cfg, budget_s: float = 12.0):
    """The fp64 oracle as it stands, on a bounded sample of the workload's query rows."""
    import oracle
    threads = oracle.threads()
    if isinstance(cfg, W.DSAConfig):
        rows_all = list(range(cfg.rows))
        what = "query rows" if cfg.prefill_start < 0 else "query tokens"

        def timed(n_threads, budget):
            oracle.set_threads(n_threads)
            t0 = time.perf_counter()
            oracle.dsa_step(inp, rows_all[:1], with_scores=False)
            one = time.perf_counter() - t0
            n = int(max(1, min(len(rows_all), n_threads * 4, n_threads * (budget // max(one, 1e-3)))))
            t0 = time.perf_counter()
            oracle.dsa_step(inp, rows_all[:n], with_scores=False)
            return n, time.perf_counter() - t0

        n, dt = timed(threads, budget_s)
        n1, dt1 = timed(1, budget_s * 0.6)
        oracle.set_threads(threads)
        unit_n = n
        sample = f"{n} of {cfg.rows} {what} of the workload (indexer over every visible key, top-{cfg.topk}, sparse MLA)"
        return {"value": unit_n / dt, "cores": threads, "kind": "oracle", "sample": sample, "seconds": round(dt, 3),
                "one_core": {"value": n1 / dt1, "cores": 1, "seconds": round(dt1, 3),
                             "sample": f"{n1} of {cfg.rows} {what}, the same oracle limited to one host thread"}}
    elif isinstance(cfg, W.CSAConfig):
        t0 = time.perf_counter()
        oracle.csa_step(inp, [0])
        one = time.perf_counter() - t0
        n = int(max(1, min(cfg.n_seqs, budget_s // max(one, 1e-3))))
        t0 = time.perf_counter()
        oracle.csa_step(inp, list(range(n)))
        dt = time.perf_counter() - t0
        unit_n = n
        sample = (f"{n} of {cfg.n_seqs} query rows (compression of the whole history inside the timed call, "
                  f"indexer over every compressed key, top-{cfg.topk}, attention)")
        threads = 1
    elif isinstance(cfg, W.NSAConfig):
        pairs = [(b, g) for b in range(cfg.B) for g in range(cfg.H_kv)]
        t0 = time.perf_counter()
        oracle.nsa_step(inp, pairs[:1])
        one = time.perf_counter() - t0
        n = int(max(1, min(len(pairs), budget_s // max(one, 1e-3))))
        t0 = time.perf_counter()
        oracle.nsa_step(inp, pairs[:n])
        dt = time.perf_counter() - t0
        unit_n = n / cfg.H_kv  # queries = sequences; one query spans every head
        sample = (f"{n} of {cfg.B * cfg.H_kv} (sequence, KV head) groups ({cfg.G} query heads each; "
                  f"compressed cache built inside the timed call)")
    else:
        pairs = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
        t0 = time.perf_counter()
        oracle.block_step(inp, pairs[:1])
        one = time.perf_counter() - t0
        n = int(max(1, min(len(pairs), budget_s // max(one, 1e-3))))
        t0 = time.perf_counter()
        oracle.block_step(inp, pairs[:n])
        dt = time.perf_counter() - t0
        unit_n = n / cfg.H  # queries = sequences; one query spans H heads
        sample = f"{n} of {cfg.B * cfg.H} (sequence, head) pairs"
    return {"value": unit_n / dt, "cores": threads, "kind": "oracle", "sample": sample, "seconds": round(dt, 3)}


def workload(name: str, profile_rows: int = 0):
    """The named workload; with profile_rows > 0, only its first query rows
    (decode: sequences; prefill: chunk tokens; block/NSA/CSA: sequences), a
    smaller case of the same kernels for profiler captures."""
    from dataclasses import replace
    if name in W.DSA_CONFIGS:
        cfg = W.DSA_CONFIGS[name]
        if profile_rows > 0:
            n = min(profile_rows, cfg.rows)
            if cfg.prefill_start >= 0:
                cfg = replace(cfg, name=f"{cfg.name} (first {n} queries)", rows=n)
            else:
                cfg = replace(cfg, name=f"{cfg.name} (first {n} sequences)", n_seqs=n, rows=n, lens=cfg.lens[:n])
        return cfg
    if name in W.NSA_CONFIGS:
        cfg = W.NSA_CONFIGS[name]
        return replace(cfg, B=min(profile_rows, cfg.B)) if profile_rows > 0 else cfg
    if name in W.CSA_CONFIGS:
        cfg = W.CSA_CONFIGS[name]
        return replace(cfg, n_seqs=min(profile_rows, cfg.n_seqs)) if profile_rows > 0 else cfg
    cfg = W.BLOCK_CONFIGS[name]
    return replace(cfg, B=min(profile_rows, cfg.B)) if profile_rows > 0 else cfg


def describe(cfg, flush_note):
    if isinstance(cfg, W.DSAConfig):
        kind = "prefill chunk" if cfg.prefill_start >= 0 else "decode"
        lens = (f"L={cfg.lens[0]}" if len(set(cfg.lens)) == 1 else
                f"L_b in [{min(cfg.lens)},{max(cfg.lens)}] (sum {sum(cfg.lens)}), 64-token pages, shuffled page table")
        return {"workload": f"{cfg.name} {kind}: {cfg.rows} queries, {lens}, indexer H^I={cfg.H_I} d^I={cfg.d_I} "
                            f"{cfg.idx_dtype}, top-{cfg.topk}, sparse MLA {cfg.H} heads d_c={cfg.d_c} d_R={cfg.d_R} bf16",
                "batch": cfg.rows, "seq_len": max(cfg.lens), "topk": cfg.topk, "heads": cfg.H, "l2": flush_note}
    if isinstance(cfg, W.CSAConfig):
        return {"workload": f"CSA decode: {cfg.n_seqs} queries, L={cfg.L} raw tokens compressed {cfg.m}:1 "
                            f"({cfg.n_c} entries), indexer H^I={cfg.H_I} d^I={cfg.d_I} e4m3 over the entries, "
                            f"top-{cfg.topk} + {cfg.window}-token raw window, attention {cfg.H} heads over "
                            f"{cfg.c}-wide bf16 entries (keys = values)",
                "batch": cfg.n_seqs, "seq_len": cfg.L, "topk": cfg.topk, "heads": cfg.H, "l2": flush_note}
    if isinstance(cfg, W.NSAConfig):
        return {"workload": f"NSA three-branch decode: B={cfg.B}, L={cfg.L}, {cfg.H} query heads in {cfg.H_kv} GQA "
                            f"groups, head_dim {cfg.D} bf16, block {cfg.block} (compression = selection blocks), "
                            f"top-{cfg.top_blocks} blocks chosen per group, {cfg.window}-token window, fp32 gates",
                "batch": cfg.B, "seq_len": cfg.L, "heads": cfg.H, "kv_heads": cfg.H_kv, "l2": flush_note}
    return {"workload": f"block-sparse decode: B={cfg.B}, L={cfg.L}, {cfg.H} MHA heads, head_dim {cfg.D} bf16, "
                        f"block {cfg.block}, top-{cfg.top_blocks} + {cfg.sink_blocks} sink block + {cfg.window}-token window",
            "batch": cfg.B, "seq_len": cfg.L, "heads": cfg.H, "l2": flush_note}


def make_step(cfg, dev, rank, sa, topk_path: str = "scores", out_dtype=torch.bfloat16):
    """Seeded inputs of a workload (each rank its own seed) and its step."""
    if isinstance(cfg, W.DSAConfig):
        inp = W.dsa_inputs(cfg, dev, seed=rank_seed(cfg.seed, rank))
        return inp, DecodeStep(inp, sa, topk_path, out_dtype)
    if isinstance(cfg, W.NSAConfig):
        inp = W.nsa_inputs(cfg, dev, seed=rank_seed(cfg.seed, rank))
        return inp, NsaStep(inp, sa)
    if isinstance(cfg, W.CSAConfig):
        inp = W.csa_inputs(cfg, dev, seed=rank_seed(cfg.seed, rank))
        return inp, CsaStep(inp, sa, out_dtype)
    inp = W.block_inputs(cfg, dev, seed=rank_seed(cfg.seed, rank))
    return inp, BlockStep(inp, sa)


def measure(cfg, args, dev, local, rank, ws, sa, flush, config_key):
    """Warm-up, then the timed steps (graph replays), the per-stage steps and
    the end-to-end steps of one workload; returns the result fields of its
    JSON line (without the top-level run keys) and the inputs."""
    inp, step = make_step(cfg, dev, rank, sa, args.topk_path,
                          torch.bfloat16 if args.out_dtype == "bf16" else torch.float32)
    for _ in range(args.warmup):
        flush.zero_()
        step.indexer()
        step.rest()
    torch.cuda.synchronize()
    if sa.check_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    kept = step.kept_candidates() if isinstance(step, DecodeStep) else 0

    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    graph = capture_step(step)
    with ClockSampler(local) as clk:
        # the step: one graph replay each (the stage events of time_steps add
        # gaps between kernels); the stages: separate event-bracketed steps
        graph_ms = time_graph(graph, args.steps, flush) if graph is not None else None
        step_ms, stage_ms = time_steps(step, args.steps, flush)
    if graph_ms is not None:
        step_ms = graph_ms
    del graph
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # L2 flushed inside the end-to-end loop only where a step's working set
    # fits in L2; a larger one (long decode 210 MB, CSA 214 MB, ragged, block)
    # streams through it and evicts its own data before the next step reads it
    flush_each = step_working_set(cfg, step) < L2_BYTES
    e2e_ms, h2d, d2h = e2e_steps(step, args.steps, flush, flush_each)
    err = sa.check_device_error()
    if err != 0:
        raise RuntimeError(f"device error word 0x{err:x}")

    ms = statistics.mean(step_ms)
    t_idx, t_topk, t_attn = (statistics.mean(x) for x in stage_ms)
    e2e = statistics.mean(e2e_ms)
    ms, t_idx, t_topk, t_attn, e2e = reduce_max([ms, t_idx, t_topk, t_attn, e2e], ws, dev)
    first = t_idx

    hbm, bf16_burst, bf16_sus, peak_src = peaks()
    res = {}
    if isinstance(cfg, W.DSAConfig):
        prefill = cfg.prefill_start >= 0
        units = cfg.rows * ws
        unit = "tokens/s" if prefill else "queries/s"
        metric = "sparse-MLA prefill tokens/s (indexer+topk+attn)" if prefill else DECODE_METRIC
        keys_b, rows_b = decode_bytes(cfg)
        score_b = int(cfg.n_visible().sum()) * 4
        if prefill:
            # a compute-bound chunk: both big kernels are contractions, so they
            # are reported against the tensor pipe (the sustained peak: the
            # chunk lasts milliseconds); fp8 = 2x bf16 (nominal ratio)
            fi, fm = prefill_flops(cfg)
            kern = {
                "indexer": {"kernel": "idx_tc_kernel", "us": t_idx * 1e3, "flop": fi, "peak_tflops": bf16_sus * 2.0,
                            "peak_source": f"{peak_src} bf16 sustained x 2 (nominal fp8/bf16 ratio)"},
                "topk": {"kernel": "topk_kernel", "us": t_topk * 1e3, "bytes": score_b},
                "attn": {"kernel": "mla_kernel", "us": t_attn * 1e3, "flop": fm, "peak_tflops": bf16_sus,
                         "peak_source": f"{peak_src} bf16 sustained"},
            }
            for v in kern.values():
                if "flop" in v:
                    v["tflops"] = round(v["flop"] / (v["us"] * 1e-6) / 1e12, 1)
                    v["tensor_frac"] = round(v["tflops"] / v["peak_tflops"], 4)
                else:
                    v["hbm_gbs"] = round(v["bytes"] / (v["us"] * 1e-6) / 1e9, 1)
                    v["hbm_frac"] = round(v["hbm_gbs"] / hbm, 4)
                v["us"] = round(v["us"], 2)
            dom_name = max(("indexer", "attn"), key=lambda n: kern[n]["us"])
            dom = kern[dom_name]
            roof = {"bound": "tensor", "achieved": dom["tflops"], "peak": dom["peak_tflops"], "unit": "TFLOP/s",
                    "frac": dom["tensor_frac"], "traffic": None, "kernel": dom["kernel"],
                    "peak_source": dom["peak_source"]}
        else:
            if step.cand_path:
                # the indexer keeps candidates instead of writing every score;
                # the Top-K reads the first-digit counts and the candidates
                kern = {
                    "indexer": {"kernel": "idx_tc_kernel (candidates)", "us": t_idx * 1e3, "bytes": keys_b},
                    "topk": {"kernel": "topk_cand_kernel", "us": t_topk * 1e3,
                             "bytes": cfg.rows * 4096 * 4 + kept * 8, "candidates_per_step": kept},
                    "attn": {"kernel": "mla_kernel (+ mla_combine_kernel)", "us": t_attn * 1e3, "bytes": rows_b},
                }
            else:
                kern = {
                    "indexer": {"kernel": "idx_tc_kernel" if cfg.idx_dtype == "e4m3" else "idx_cc_kernel",
                                "us": t_idx * 1e3, "bytes": keys_b},
                    "topk": {"kernel": "topk_kernel", "us": t_topk * 1e3, "bytes": score_b},
                    "attn": {"kernel": "mla_kernel (+ mla_combine_kernel)", "us": t_attn * 1e3, "bytes": rows_b},
                }
            for v in kern.values():
                v["hbm_gbs"] = round(v["bytes"] / (v["us"] * 1e-6) / 1e9, 1)
                v["hbm_frac"] = round(v["hbm_gbs"] / hbm, 4)
                v["us"] = round(v["us"], 2)
            dom_name = max(kern, key=lambda n: kern[n]["us"])
            dom = kern[dom_name]
            tr = TRAFFIC.get(config_key, {}) if not args.profile_rows else {}  # records are of the full workloads
            traffic = None
            if tr.get("bytes_per_launch") and tr.get("stage") == dom_name and tr.get("src_sha") == src_sha(
                    "sparse_attention_07_b200/csrc/" + tr.get("kernel", "")):
                traffic = tr["bytes_per_launch"]
            roof = {"bound": "hbm", "achieved": dom["hbm_gbs"], "peak": hbm, "unit": "GB/s",
                    "frac": dom["hbm_frac"], "traffic": traffic, "kernel": dom["kernel"],
                    "peak_source": f"{peak_src} hbm_gbs"}
            step_gbs = (keys_b + rows_b) / (ms * 1e-3) / 1e9
            res["step_roofline"] = {"bytes_per_step": keys_b + rows_b, "indexer_key_bytes": keys_b,
                                    "gathered_row_bytes": rows_b, "achieved": round(step_gbs, 1), "peak": hbm,
                                    "unit": "GB/s", "frac": round(step_gbs / hbm, 4),
                                    "peak_source": f"{peak_src} hbm_gbs"}
        res["kernels"] = kern
        if not prefill and config_key == "long":
            res["projections"] = time_projections(step, min(args.steps, 20), flush, hbm)
    elif isinstance(cfg, W.CSAConfig):
        units = cfg.n_seqs * ws
        unit = "queries/s"
        metric = "CSA decode queries/s (indexer over compressed entries + topk + window + attention)"
        keys_b, rows_b = csa_bytes(cfg)
        kern = {"indexer": {"kernel": "idx_tc_kernel", "us": t_idx * 1e3, "bytes": keys_b},
                "topk": {"kernel": "topk_kernel", "us": t_topk * 1e3, "bytes": cfg.n_seqs * cfg.n_c * 4},
                "attn": {"kernel": "csa_window_index_kernel + mla_kernel (+ combine)", "us": t_attn * 1e3,
                         "bytes": rows_b}}
        for v in kern.values():
            v["hbm_gbs"] = round(v["bytes"] / (v["us"] * 1e-6) / 1e9, 1)
            v["hbm_frac"] = round(v["hbm_gbs"] / hbm, 4)
            v["us"] = round(v["us"], 2)
        dom = kern[max(kern, key=lambda n: kern[n]["us"])]
        roof = {"bound": "hbm", "achieved": dom["hbm_gbs"], "peak": hbm, "unit": "GB/s", "frac": dom["hbm_frac"],
                "traffic": None, "kernel": dom["kernel"], "peak_source": f"{peak_src} hbm_gbs"}
        step_gbs = (keys_b + rows_b) / (ms * 1e-3) / 1e9
        res["step_roofline"] = {"bytes_per_step": keys_b + rows_b, "achieved": round(step_gbs, 1), "peak": hbm,
                                "unit": "GB/s", "frac": round(step_gbs / hbm, 4)}
        res["kernels"] = kern
        res["compression"] = time_compress(step, min(args.steps, 10), flush, hbm)
    elif isinstance(cfg, W.NSAConfig):
        units = cfg.B * ws
        unit = "queries/s"
        metric = "NSA decode queries/s (compression + group block choice + selection + window, gated)"
        nbytes = nsa_bytes(cfg)
        ach = nbytes / (first * 1e-3) / 1e9
        tr = TRAFFIC.get(config_key, {}) if not args.profile_rows else {}  # records are of the full workloads
        traffic = tr.get("bytes_per_launch") if tr.get("src_sha") == src_sha(
            "sparse_attention_07_b200/csrc/" + tr.get("kernel", "nsa.cu")) else None
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
                "traffic": traffic, "kernel": "nsa_decode_kernel", "bytes_per_launch": nbytes,
                "peak_source": f"{peak_src} hbm_gbs"}
    else:
        units = cfg.B * ws
        unit = "queries/s"
        metric = "block-sparse decode queries/s (pooled-block scan+top-k+block attention)"
        nbytes, u_tokens = block_bytes(cfg, step.union_tokens)
        ach = nbytes / (first * 1e-3) / 1e9
        tr = TRAFFIC.get(config_key, {}) if not args.profile_rows else {}  # records are of the full workloads
        traffic = tr.get("bytes_per_launch") if tr and tr.get("src_sha") == src_sha(
            "sparse_attention_07_b200/csrc/" + tr.get("kernel", "block_sparse.cu")) else None
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
                "traffic": traffic, "kernel": "block_sparse_cluster_kernel", "bytes_per_launch": nbytes,
                "union_tokens": u_tokens, "peak_source": f"{peak_src} hbm_gbs"}
    value = units / (ms * 1e-3)
    res.update({
        "metric": metric, "value": round(value, 1), "unit": unit, "ms_per_step": round(ms, 5),
        "config": dict(describe(cfg, f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, outside the events)"),
                       timing=("step: one CUDA-graph replay of the step's launches per timed step; stage times: "
                               "the same number of stream-launched steps with an event between stages"
                               if graph_ms is not None else
                               "step and stage times: stream-launched steps with an event between stages")),
        "roofline": roof,
        "e2e": {"value": round(units / (e2e * 1e-3), 1), "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "timing": (f"{args.steps} steps in one event pair, up to {E2E_SLOTS} in flight: copy-in, compute "
                           "and copy-out streams; per step the inputs are copied in from pinned host memory "
                           "(one packed transfer), moved to the step's tensors, "
                           + ("L2 is flushed (working set under the L2 size), " if flush_each else
                              f"no flush (working set {step_working_set(cfg, step) / 1e6:.0f} MB, over the "
                              f"{L2_BYTES / 1e6:.0f} MB L2), ")
                           + "the step runs and its output is read back to pinned host memory")},
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": clk.summary(),
    })
    if isinstance(step, (DecodeStep, CsaStep)):
        res["config"]["attention_output"] = ("bf16 (fp32 softmax and accumulation, rounded once)"
                                             if step.out.dtype == torch.bfloat16 else "fp32")
    if isinstance(step, DecodeStep):
        res["config"]["indexer_output"] = ("Top-K candidates (keys at or above a proven bound on the row's k-th "
                                           "largest)" if step.cand_path else "every score")
    if ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(inp, cfg)
        res["cpu_baseline"]["unit"] = unit
    del step
    return res, inp


def run_native(args):
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import sparse_attention_07_b200 as sa
    sa.lib()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    cfg = workload(args.config, args.profile_rows)
    main_res, inp = measure(cfg, args, dev, local, rank, ws, sa, flush, args.config)
    del inp
    res = {"impl": "native"}
    res.update(main_res)
    res.update({"n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None,
                "dtype": "e4m3 indexer / bf16 MLA, fp32 accumulate" if isinstance(cfg, (W.DSAConfig, W.CSAConfig))
                else "bf16, fp32 accumulate",
                "data": "synthetic (seeded, shapes and value distributions of the workload)"})
    if args.config == "long" and not args.no_l128k and args.profile_rows == 0:
        # the metric's second length: the ragged workload (64 rows, histories
        # 8K-128K in shuffled 64-token pages), measured the same way
        torch.cuda.empty_cache()
        gate, inp = measure(W.RAGGED, args, dev, local, rank, ws, sa, flush, "ragged")
        del inp
        gate.pop("metric", None)
        res["l128k"] = gate
    if rank == 0:
        print(json.dumps(res), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


# history lengths of the dual-mode measurement (long-decode shapes otherwise)
CROSSOVER_L = (1024, 2048, 3072, 4096, 6144, 8192, 12288, 16384)


def run_crossover(args):
    """Short-sequence mode vs DSA: the step time of the DSA path (indexer ->
    Top-K -> sparse MLA) and of dense MLA over every visible position, for the
    long-decode shapes at growing history lengths; `value` is the length above
    which DSA is faster (linear interpolation between measured lengths)."""
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import sparse_attention_07_b200 as sa
    sa.lib()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    table = []
    launches = 0
    for L in CROSSOVER_L:
        cfg = W.small_dsa(W.LONG, lens=(L,) * W.LONG.n_seqs)
        inp = W.dsa_inputs(cfg, dev, seed=rank_seed(cfg.seed + L, rank))
        dsa = DecodeStep(inp, sa)
        nv = inp["n_visible"]
        out = torch.empty(cfg.rows, cfg.H, cfg.d_c, dtype=torch.float32, device=dev)
        wsd = torch.empty(sa.dense_mla_workspace_size(cfg.rows, cfg.H, L, cfg.d_c), dtype=torch.uint8, device=dev)

        def dense():
            sa.dense_mla_decode(inp["q_lat"], inp["q_rope"], inp["c_cache"], inp["kr_cache"], nv, L, cfg.scale,
                                cfg.pages_per_seq, page_table=inp["page_table"], out=out, workspace=wsd)

        def time_fn(fn):
            for _ in range(args.warmup):
                flush.zero_()
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for a, b in ev:
                flush.zero_()
                a.record()
                fn()
                b.record()
            torch.cuda.synchronize()
            return statistics.mean(a.elapsed_time(b) for a, b in ev)

        t_dsa = time_fn(lambda: (dsa.indexer(), dsa.rest()))
        t_dense = time_fn(dense)
        launches += args.steps * (dsa.launches_per_step + 1 + (1 if sa.dense_mla_workspace_size(
            cfg.rows, cfg.H, L, cfg.d_c) > 0 else 0))
        table.append({"L": L, "dsa_us": round(t_dsa * 1e3, 2), "dense_us": round(t_dense * 1e3, 2)})
        del inp, dsa, wsd
        torch.cuda.empty_cache()
    if sa.check_device_error() != 0:
        raise RuntimeError("device error word set")
    cross = None
    for a, b in zip(table, table[1:]):
        da, db = a["dsa_us"] - a["dense_us"], b["dsa_us"] - b["dense_us"]
        if da >= 0 > db:
            cross = round(a["L"] + (b["L"] - a["L"]) * da / (da - db))
            break
    if cross is None and table and table[0]["dsa_us"] < table[0]["dense_us"]:
        cross = table[0]["L"]
    hbm, _, _, peak_src = peaks()
    last = table[-1]
    dense_bytes = W.LONG.n_seqs * last["L"] * (W.LONG.d_c + W.LONG.d_R) * 2
    ach = dense_bytes / (last["dense_us"] * 1e-6) / 1e9
    res = {
        "impl": "native", "metric": "DSA vs dense MLA decode crossover (history length above which DSA is faster)",
        "value": cross, "unit": "tokens", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": None, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 indexer / bf16 MLA, fp32 accumulate", "data": "synthetic (seeded)",
        "config": {"workload": "long-decode shapes (32 queries, H^I=64 e4m3, top-2048, 128-head MLA) at history "
                               "lengths " + ",".join(str(x) for x in CROSSOVER_L),
                   "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, outside the events)"},
        "crossover": table,
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
                     "traffic": None, "kernel": f"mla_kernel, dense mode at L={last['L']}",
                     "peak_source": f"{peak_src} hbm_gbs"},
        "e2e": None, "gpu_launches": launches,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)


def run_reference(args):
    """The oracle as the reference arm, timed on the host cores."""
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import oracle
    cfg = workload(args.config)
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    if isinstance(cfg, W.DSAConfig):
        inp = W.dsa_inputs(cfg, dev, seed=cfg.seed)
        prefill = cfg.prefill_start >= 0
        unit = "tokens/s" if prefill else "queries/s"
        metric = "sparse-MLA prefill tokens/s (indexer+topk+attn)" if prefill else DECODE_METRIC
        t0 = time.perf_counter()
        oracle.dsa_step(inp, [0], with_scores=False)
        one = time.perf_counter() - t0
        per_step = max(1, min(cfg.rows, oracle.threads(), int(150.0 / max(1, args.steps + args.warmup) / max(one, 1e-3))))
        rows = list(range(per_step))
        run = lambda: oracle.dsa_step(inp, rows, with_scores=False)  # noqa: E731
        units_per_step = per_step
        sample = f"{per_step} query rows of the workload per step"
    elif isinstance(cfg, W.CSAConfig):
        inp = W.csa_inputs(cfg, dev, seed=cfg.seed)
        unit = "queries/s"
        metric = "CSA decode queries/s (indexer over compressed entries + topk + window + attention)"
        run = lambda: oracle.csa_step(inp, [0])  # noqa: E731
        units_per_step = 1
        sample = "one query row per step (compression of its whole history inside the timed call)"
    elif isinstance(cfg, W.NSAConfig):
        inp = W.nsa_inputs(cfg, dev, seed=cfg.seed)
        unit = "queries/s"
        metric = "NSA decode queries/s (compression + group block choice + selection + window, gated)"
        run = lambda: oracle.nsa_step(inp, [(0, 0)])  # noqa: E731
        units_per_step = 1.0 / cfg.H_kv  # one of the query's KV-head groups
        sample = (f"one (sequence, KV head) group ({cfg.G} of the query's {cfg.H} heads) per step, compressed cache "
                  f"built inside the timed call")
    else:
        inp = W.block_inputs(cfg, dev, seed=cfg.seed)
        unit, metric = "queries/s", "block-sparse decode queries/s (pooled-block scan+top-k+block attention)"
        pairs = [(0, h) for h in range(cfg.H)]
        run = lambda: oracle.block_step(inp, pairs)  # noqa: E731
        units_per_step = 1
        sample = f"one sequence ({cfg.H} heads) per step"
    for _ in range(args.warmup):
        run()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    value = units_per_step / (ms * 1e-3)
    print(json.dumps({
        "impl": "reference", "metric": metric, "value": round(value, 3), "unit": unit, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": describe(cfg, "n/a (host)"),
        "cpu_baseline": {"value": round(value, 3), "unit": unit, "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--config", default="long",
                   choices=sorted(list(W.DSA_CONFIGS) + list(W.BLOCK_CONFIGS) + list(W.NSA_CONFIGS) +
                                  list(W.CSA_CONFIGS) + ["crossover"]))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--out-dtype", choices=["bf16", "f32"], default="bf16",
                   help="DSA / CSA: storage type of the attention output (the step's result)")
    p.add_argument("--topk-path", choices=["cand", "scores"], default="scores",
                   help="decode: the indexer keeps Top-K candidates (cand) or writes every score (scores)")
    p.add_argument("--no-l128k", action="store_true",
                   help="long decode only: skip the nested L=128K (ragged) measurement")
    p.add_argument("--profile-rows", type=int, default=0,
                   help="profiler captures: run only the first N query rows / sequences of the workload")
    args = p.parse_args(argv)
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    if args.config == "crossover":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the crossover mode times two GPU paths; "
                              "the oracle arm covers the workload configs"}), flush=True)
        else:
            run_crossover(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
