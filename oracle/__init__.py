"""fp64 CPU oracle for the sparse-attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
(``sparse_attention_07_b200``) never imports, links or calls it, and the two
share no code: the only module both read is ``workloads`` (seeded inputs, no
arithmetic of the method).

The heavy loops live in ``sa_oracle.c`` (plain C, double precision, built by
``build()`` below with gcc + OpenMP over independent queries).  This file
converts inputs to float64 (bf16, fp8 e4m3 and fp32 values are all exact in
fp64; the conversion is torch's CPU cast), looks up pages, and holds the small
numpy helpers the pins use.  Each function cites the passage it follows:

  [Notes]  "Sparse Attention 数学学习笔记" (echobase-5bl.pages.dev, 2026.09.14)
  [MLA-S]  "MLA 与稀疏注意力：少存一点，还是少看一点？" (tianyi-zhang-02.github.io)
  [Ch11]   "第 11 章 稀疏注意力" (book.shippingwang.com)
  [LLMRes] "LLM注意力优化：稀疏注意力" (wln20.github.io)

Parity status: every function here is pinned by a test in
``tests/test_oracle_pins.py``; none is "parity unpinned", except the block
selection of near-tied blocks, which fp64 and fp32 may order differently (the
GPU tests accept a differing block only when its score is within the stated
tolerance of the boundary score).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsa_oracle.so")
_lib = None

PAGE = 64


def build(force: bool = False) -> str:
    """Compile sa_oracle.c into libsa_oracle.so (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        D = ctypes.c_double
        lib.sa_oracle_index_scores.argtypes = [I, I, I, P, P, P, P, P, P, I64]
        lib.sa_oracle_topk.argtypes = [I, P, I64, P, I, P]
        lib.sa_oracle_sparse_mla.argtypes = [I, I, I, I, P, P, P, P, P, I, D, P, P]
        lib.sa_oracle_block_mean_pool.argtypes = [I, I, I, P, P]
        lib.sa_oracle_block_sparse.argtypes = [I, I, I, I, I, I, D, P, P, P, P, P, P]
        lib.sa_oracle_block_attend.argtypes = [I, I, I, P, I, I, I, D, P, P, P, P]
        lib.sa_oracle_threads.restype = I
        lib.sa_oracle_set_threads.argtypes = [I]
        _lib = lib
    return _lib


def threads() -> int:
    """Host threads the C oracle runs on (OpenMP)."""
    return int(_load().sa_oracle_threads())


def set_threads(n: int) -> None:
    """Limit the C oracle to n host threads (n >= 1)."""
    _load().sa_oracle_set_threads(int(n))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# C-backed definitions

def index_scores(q, w, keys, key0, n_vis, out_ld: Optional[int] = None) -> np.ndarray:
    """Lightning-indexer scores, [Notes] §9 (I_{t,s}) / [MLA-S] DSA section.

    q [rows,H_I,d_I], w [rows,H_I], keys [n_keys,d_I] (each sequence in logical
    order), key0[r] = index in ``keys`` of the row's position 0, n_vis[r] =
    visible positions.  Returns [rows, out_ld] float64; entries s >= n_vis[r]
    are NaN.
    """
    q, w, keys = _f64(q), _f64(w), _f64(keys)
    key0, n_vis = _i64(key0), _i64(n_vis)
    rows, H_I, d_I = q.shape
    out_ld = int(out_ld if out_ld is not None else (n_vis.max() if rows else 0))
    out = np.full((rows, max(out_ld, 1)), np.nan)
    _load().sa_oracle_index_scores(rows, H_I, d_I, _ptr(q), _ptr(w), _ptr(keys), _ptr(key0),
                                   _ptr(n_vis), _ptr(out), out.shape[1])
    return out[:, :out_ld]


def topk(scores, n_valid, k: int) -> np.ndarray:
    """Exact Top-K, [Notes] §9 and [MLA-S] ``selected_positions`` order.

    Keeps the min(k, n) positions with the largest score, equal scores going to
    the lower position; returns them ascending, padded with -1 to k.
    """
    s = _f64(scores)
    if s.ndim == 1:
        s = s[None]
    n_valid = _i64(np.broadcast_to(np.asarray(n_valid), (s.shape[0],)))
    out = np.empty((s.shape[0], k), dtype=np.int32)
    _load().sa_oracle_topk(s.shape[0], _ptr(s), s.shape[1], _ptr(n_valid), k, _ptr(out))
    return out


def sparse_mla(q_lat, q_rope, c, kr, sel, scale: float):
    """Sparse MLA latent attention, [MLA-S] full-score section + [Notes] §2/§8.

    q_lat [rows,H,d_c] (absorbed), q_rope [rows,H,d_R], c [n,d_c], kr [n,d_R],
    sel [rows,k] row of c/kr per selected slot (-1 = empty).  Returns
    (out [rows,H,d_c] = sum_j a_j c_j, lse [rows,H] natural log).
    """
    q_lat, q_rope, c, kr = _f64(q_lat), _f64(q_rope), _f64(c), _f64(kr)
    sel = _i64(sel)
    rows, H, d_c = q_lat.shape
    d_R = q_rope.shape[2]
    k = sel.shape[1]
    out = np.zeros((rows, H, d_c))
    lse = np.zeros((rows, H))
    _load().sa_oracle_sparse_mla(rows, H, d_c, d_R, _ptr(q_lat), _ptr(q_rope), _ptr(c), _ptr(kr),
                                 _ptr(sel), k, float(scale), _ptr(out), _ptr(lse))
    return out, lse


def block_mean_pool(K, block: int) -> np.ndarray:
    """Mean of each complete block of keys, [Ch11] §12.6 (k_blocks.mean)."""
    K = _f64(K)
    L, D = K.shape
    out = np.zeros((L // block, D))
    _load().sa_oracle_block_mean_pool(L, D, block, _ptr(K), _ptr(out))
    return out


def block_sparse(q, K, V, block: int, top_blocks: int, sink_blocks: int, window: int, scale: float):
    """Block-sparse decode for one (sequence, head), [Ch11] §12.5-12.6 + [LLMRes] MoBA.

    Returns (out [D], chosen blocks [top_blocks] ascending -1 padded,
    block scores [L//block]).
    """
    q, K, V = _f64(q), _f64(K), _f64(V)
    L, D = K.shape
    out = np.zeros(D)
    sel = np.empty(top_blocks, dtype=np.int32)
    bs = np.zeros(max(L // block, 1))
    _load().sa_oracle_block_sparse(L, D, block, top_blocks, sink_blocks, window, float(scale),
                                   _ptr(q), _ptr(K), _ptr(V), _ptr(out), _ptr(sel), _ptr(bs))
    return out, sel, bs[: L // block]


def block_attend(q, K, V, chosen_blocks, block: int, sink_blocks: int, window: int, scale: float):
    """Attention over the union of given chosen blocks, sink and window
    ([Ch11] §12.5 block gather, [Notes] §2 softmax over the chosen set)."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    L, D = K.shape
    ch = np.ascontiguousarray(np.asarray(chosen_blocks, dtype=np.int32))
    out = np.zeros(D)
    _load().sa_oracle_block_attend(L, D, block, _ptr(ch), len(ch), sink_blocks, window, float(scale),
                                   _ptr(q), _ptr(K), _ptr(V), _ptr(out))
    return out


# --------------------------------------------------------------------------
# numpy helpers used by the pins

def dense_attention(q, K, V, scale: float):
    """[Notes] §1: o = sum_j softmax_j(q.k_j * scale) v_j over all positions."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    s = K @ q * scale
    a = np.exp(s - s.max())
    a /= a.sum()
    return a @ V, a


def masked_attention(scores, values, visible):
    """[Notes] §3: softmax(S + M) with M = 0 on the visible set, -inf elsewhere;
    the mask enters before the softmax ([MLA-S] masked_scalar_attention)."""
    s = _f64(scores)
    vis = np.asarray(visible, dtype=bool)
    if s.shape != vis.shape or not vis.any():
        raise ValueError("expected equal lengths and at least one visible position")
    m = np.where(vis, 0.0, -np.inf)
    z = s + m
    a = np.exp(z - z[vis].max())
    a /= a.sum()
    return float(a @ _f64(values))


def absorb(U_K, q):
    """[MLA-S] absorbed query: q^T U_K c = (U_K^T q)^T c."""
    return _f64(U_K).T @ _f64(q)


def up_project(U_V, o_lat):
    """[MLA-S] "“吸收矩阵”是交换线性计算的顺序": the output of a head is
    U_V applied to its latent aggregate, o_h = U_V,h (sum_j a_j c_j), which
    equals sum_j a_j (U_V,h c_j).  U_V [H, d_v, d_c], o_lat [rows, H, d_c]
    -> [rows, H, d_v] float64."""
    U, o = _f64(U_V), _f64(o_lat)
    rows, H, _ = o.shape
    out = np.zeros((rows, H, U.shape[1]))
    for r in range(rows):
        for h in range(H):
            out[r, h] = U[h] @ o[r, h]
    return out


def mla_chain(q_c, U_K, U_V, q_rope, c, kr, sel, scale: float):
    """The absorbed MLA decode of [MLA-S] end to end: per head the absorbed
    query U_K,h^T q^C_h (absorb), sparse MLA over the selected latent rows
    (sparse_mla), then the up-projection U_V,h (up_project).
    q_c [rows, H, d_C], U_K [H, d_C, d_c], U_V [H, d_v, d_c], q_rope
    [rows, H, d_R], c [n, d_c], kr [n, d_R], sel [rows, k] (-1 = empty).
    Returns [rows, H, d_v] float64."""
    qc, Uk = _f64(q_c), _f64(U_K)
    rows, H, _ = qc.shape
    q_lat = np.zeros((rows, H, Uk.shape[2]))
    for r in range(rows):
        for h in range(H):
            q_lat[r, h] = absorb(Uk[h], qc[r, h])
    o_lat, _ = sparse_mla(q_lat, q_rope, c, kr, sel, scale)
    return up_project(U_V, o_lat)


def dense_mass(alpha_dense, selected) -> float:
    """[Notes] §6: Z_i = sum_{j in S_i} alpha_ij."""
    a = _f64(alpha_dense)
    return float(a[np.asarray(selected, dtype=np.int64)].sum())


def error_bound(v_max: float, Z: float) -> float:
    """[Notes] §6: ||o^dense - o^sparse|| <= 2 V_max (1 - Z_i)."""
    return 2.0 * v_max * (1.0 - Z)


# --------------------------------------------------------------------------
# NSA three-branch decode ([MLA-S] "三条路径，各留住什么？" and "选块和合并输出，
# 实际算一遍"; [LLMRes] NSA steps 1-3).  Compression is the mean of each
# complete block of keys and of values (the pages' learned per-block transform
# has no weights here; [Ch11] §12.6 pools by the mean).

def shared_block_choice(head_probabilities, count: int):
    """[MLA-S] shared_block_choice: the heads that share a KV head add their
    block probabilities and keep the `count` best blocks, ties to the lower
    block index.  Returns the chosen block indices in rank order."""
    p = _f64(head_probabilities)
    if p.ndim != 2 or p.shape[1] == 0:
        raise ValueError("expected nonempty head distributions")
    if not 1 <= count <= p.shape[1]:
        raise ValueError("invalid selection count")
    totals = p.sum(axis=0)
    return sorted(range(p.shape[1]), key=lambda i: (-totals[i], i))[:count]


def nsa_select_scores(p_cmp, l: int, d: int, l_sel: int):
    """[MLA-S] NSA §3.3 aggregation of compression probabilities into selection
    block scores: p_sel[j] = sum_{u < l'/d} sum_{v < l/d} p_cmp[(l'/d) j + u + v]
    for compression blocks of length l and stride d and selection blocks of
    length l' (d divides both); terms past the end of p_cmp are absent."""
    p = _f64(p_cmp)
    if l % d or l_sel % d:
        raise ValueError("the stride must divide both block lengths")
    a, b = l_sel // d, l // d
    n_sel = (len(p) + a - 1) // a if len(p) else 0
    out = np.zeros(n_sel)
    for j in range(n_sel):
        for u in range(a):
            for v in range(b):
                i = a * j + u + v
                if i < len(p):
                    out[j] += p[i]
    return out


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to the even
    significand: bf16 keeps 8 significant bits (1 implicit + 7 stored) with
    the fp32 exponent range, so the step in the binade [2^e, 2^(e+1)) is
    2^(e-7) and below 2^-126 (the subnormals) it is 2^-133.  Values are
    returned as float64 holding the rounded value (finite inputs whose
    rounding stays below the bf16 maximum)."""
    x = _f64(x)
    out = np.zeros_like(x)
    nz = x != 0.0
    _, ex = np.frexp(x[nz])                      # |x| = f * 2^ex, 0.5 <= f < 1
    step_exp = np.maximum(ex.astype(np.int64) - 1, -126) - 7
    q = np.ldexp(x[nz], -step_exp)               # exact: scaling by a power of two
    out[nz] = np.ldexp(np.round(q), step_exp)    # np.round: half to even
    return out


def nsa_compress(X, block: int) -> np.ndarray:
    """The NSA compressed cache as stored: the mean of each complete block of
    rows of X [L, D] ([Ch11] §12.6 mean compression), kept in bf16 like the
    token cache it summarises, i.e. the block mean rounded to the nearest
    bf16 value (ties to even).  The mean is taken in float64: for bf16 inputs
    whose magnitudes within a block span less than 2^45 the float64 sum is
    exact, so this is the exact mean rounded once.  Returns [L // block, D]
    float64 holding bf16 values."""
    X = _f64(X)
    nb = X.shape[0] // block
    mean = X[: nb * block].reshape(nb, block, X.shape[1]).sum(axis=1) / block
    return bf16_round(mean)


def nsa_combine(o_cmp, o_sel, o_win, gates):
    """[MLA-S] g_c o_c + g_s o_s + g_w o_w with independent (sigmoid) gates:
    the gates are not normalised to sum to one."""
    g = _f64(gates)
    return g[0] * _f64(o_cmp) + g[1] * _f64(o_sel) + g[2] * _f64(o_win)


def _softmax_attend(q, K, V, scale):
    s = K @ q * scale
    a = np.exp(s - s.max())
    a /= a.sum()
    return a @ V, a


def nsa_decode_group(q, K, V, block: int, top_blocks: int, window: int, gates, scale: float, chosen=None,
                     compressed=None):
    """One decode query per head of a GQA group sharing one KV head.

    q [G, D], K/V [L, D] (the history; the query sees all L positions), gates
    [G, 3] (compression, selection, window).  Branches, each with its own
    softmax:
      compression: the complete blocks n < L // block, key mean(K_block) and
        value mean(V_block) (no block holding a position >= L is formed);
      selection: the heads' compression probabilities summed over the group
        pick min(top_blocks, n_blocks) blocks (ties to the lower index); every
        head attends to all tokens of those blocks;
      window: the last `window` positions.
    A branch with no position (no complete block) contributes zero.
    `chosen` (block indices) replaces the group's own choice when given: it
    evaluates the branches on another valid choice among near-tied blocks.
    `compressed` = (K_bar, V_bar) replaces the exact block means (e.g. with
    the stored bf16 cache of nsa_compress).
    Returns (out [G, D], chosen blocks ascending, p_cmp [G, n_blocks])."""
    q, K, V, g = _f64(q), _f64(K), _f64(V), _f64(gates)
    G, D = q.shape
    L = K.shape[0]
    nb = L // block
    if compressed is not None:
        kbar, vbar = _f64(compressed[0])[:nb], _f64(compressed[1])[:nb]
    else:
        kbar = K[: nb * block].reshape(nb, block, D).mean(axis=1) if nb else np.zeros((0, D))
        vbar = V[: nb * block].reshape(nb, block, D).mean(axis=1) if nb else np.zeros((0, D))
    p_cmp = np.zeros((G, nb))
    o_cmp = np.zeros((G, D))
    for h in range(G):
        if nb:
            o_cmp[h], p_cmp[h] = _softmax_attend(q[h], kbar, vbar, scale)
    if chosen is None:
        chosen = sorted(shared_block_choice(p_cmp, min(top_blocks, nb))) if nb and top_blocks > 0 else []
    else:
        chosen = sorted(int(c) for c in chosen)
    tokens = np.concatenate([np.arange(b * block, (b + 1) * block) for b in chosen]) if chosen else None
    w0 = max(0, L - window)
    out = np.zeros((G, D))
    for h in range(G):
        o_sel = _softmax_attend(q[h], K[tokens], V[tokens], scale)[0] if tokens is not None else np.zeros(D)
        o_win = _softmax_attend(q[h], K[w0:], V[w0:], scale)[0] if window > 0 and L > 0 else np.zeros(D)
        out[h] = nsa_combine(o_cmp[h], o_sel, o_win, g[h])
    return out, np.asarray(chosen, dtype=np.int64), p_cmp


# --------------------------------------------------------------------------
# CSA: DSA over m-token compressed entries ([LLMRes] "DeepSeek CSA & HCA";
# [MLA-S] on DeepSeek-V4's two kinds of attention layer).

def csa_compress(Ca, Cb, Za, Zb, Ba, Bb, m: int) -> np.ndarray:
    """Compressed entries of one sequence, [LLMRes] CSA.  Ca, Cb, Za, Zb
    [n, c] (the two streams of entries and their compression weights), Ba, Bb
    [m, c] (position biases).  Entry i (0 <= i < n // m, complete groups only)
    merges group i of stream a with group i - 1 of stream b: the 2m weight
    rows Za[mi : m(i+1)] + Ba and Zb[m(i-1) : mi] + Bb, stacked along the
    sequence, are normalised by a softmax along the sequence separately for
    every channel, and weight the matching 2m entry rows, summed.  For i = 0
    stream b contributes nothing (its weights are -inf, its entries 0).
    Returns [n // m, c] float64."""
    Ca, Cb, Za, Zb, Ba, Bb = (_f64(x) for x in (Ca, Cb, Za, Zb, Ba, Bb))
    n, c = Ca.shape
    nc = n // m
    out = np.zeros((nc, c))
    for i in range(nc):
        za = Za[m * i: m * (i + 1)] + Ba
        ca = Ca[m * i: m * (i + 1)]
        if i == 0:
            zb, cb = np.full((m, c), -np.inf), np.zeros((m, c))
        else:
            zb, cb = Zb[m * (i - 1): m * i] + Bb, Cb[m * (i - 1): m * i]
        z = np.concatenate([za, zb], axis=0)
        e = np.exp(z - z.max(axis=0, keepdims=True))
        wgt = e / e.sum(axis=0, keepdims=True)
        out[i] = (wgt[:m] * ca).sum(axis=0) + (wgt[m:] * cb).sum(axis=0)
    return out


def csa_attend(q, C_comp, C_raw, chosen, window: int, scale: float):
    """CSA core attention of one query, [LLMRes] CSA: every head of q [H, c]
    attends (one softmax, keys = values = the entries) to the chosen
    compressed entries C_comp[chosen] together with the raw entries of the
    last `window` positions of C_raw [L, c].  Returns [H, c]."""
    q, C_comp, C_raw = _f64(q), _f64(C_comp), _f64(C_raw)
    L = C_raw.shape[0]
    rows = [C_comp[int(j)] for j in chosen if j >= 0] + [C_raw[t] for t in range(max(0, L - window), L)]
    if not rows:
        return np.zeros_like(q)
    E = np.stack(rows)
    s = q @ E.T * scale
    a = np.exp(s - s.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)
    return a @ E


# --------------------------------------------------------------------------
# Whole-step reference on workload tensors (any device; values copied to host)

def _host64(t):
    import torch
    return t.detach().to("cpu").to(torch.float64).numpy()


def pool_rows(page_table, pages_per_seq: int, seq: int, positions) -> np.ndarray:
    """Row of the page pool holding each logical position of ``seq``."""
    pos = _i64(positions)
    page = pos // PAGE
    if page_table is None:
        phys = seq * pages_per_seq + page
    else:
        phys = np.asarray(page_table)[seq, page].astype(np.int64)
    return phys * PAGE + pos % PAGE


def dsa_step(inp: dict, rows: Sequence[int], with_scores: bool = True, with_attention: bool = True) -> dict:
    """Indexer -> Top-K -> sparse MLA for the chosen query rows of a workload.

    ``inp`` is a dict made by ``workloads.dsa_inputs``.  Returns, per chosen
    row (in the order given): ``scores`` [n_rows, L_max] (NaN past the visible
    length), ``idx`` [n_rows, k] int32 and, unless ``with_attention`` is
    False, ``out`` [n_rows,H,d_c], ``lse`` [n_rows,H] float64.
    """
    import torch
    cfg = inp["cfg"]
    rows = [int(r) for r in rows]
    table = None if inp["page_table"] is None else inp["page_table"].cpu().numpy()
    pps = cfg.pages_per_seq
    n_vis_all = inp["n_visible"].cpu().numpy().astype(np.int64)
    sor = inp["seq_of_row"]
    sor = np.arange(cfg.rows) if sor is None else sor.cpu().numpy().astype(np.int64)
    seqs = sorted({int(sor[r]) for r in rows})
    key_blocks, key0_of_seq, off = [], {}, 0
    for s in seqs:
        n = int(max(n_vis_all[r] for r in rows if sor[r] == s))
        pr = torch.from_numpy(pool_rows(table, pps, s, np.arange(n)))
        key_blocks.append(_host64(inp["k_idx_cache"][pr.to(inp["k_idx_cache"].device)]))
        key0_of_seq[s] = off
        off += n
    keys = np.concatenate(key_blocks, axis=0) if key_blocks else np.zeros((0, cfg.d_I))
    ridx = torch.tensor(rows, dtype=torch.long, device=inp["q_idx"].device)
    q = _host64(inp["q_idx"][ridx])
    w = _host64(inp["w"][ridx])
    n_vis = np.array([n_vis_all[r] for r in rows], dtype=np.int64)
    key0 = np.array([key0_of_seq[int(sor[r])] for r in rows], dtype=np.int64)
    scores = index_scores(q, w, keys, key0, n_vis, out_ld=cfg.L_max)
    idx = topk(np.nan_to_num(scores, nan=-np.inf), n_vis, cfg.topk)
    if not with_attention:
        return dict(idx=idx, scores=scores, n_visible=n_vis)
    # gather the selected latent rows of every chosen query row
    sel = np.full(idx.shape, -1, dtype=np.int64)
    flat = []
    for i, r in enumerate(rows):
        valid = idx[i] >= 0
        pr = pool_rows(table, pps, int(sor[r]), idx[i][valid])
        sel[i, valid] = np.arange(len(flat), len(flat) + len(pr))
        flat.extend(pr.tolist())
    fr = torch.tensor(flat, dtype=torch.long, device=inp["c_cache"].device)
    c = _host64(inp["c_cache"][fr]) if flat else np.zeros((0, cfg.d_c))
    kr = _host64(inp["kr_cache"][fr]) if flat else np.zeros((0, cfg.d_R))
    out, lse = sparse_mla(_host64(inp["q_lat"][ridx]), _host64(inp["q_rope"][ridx]), c, kr, sel, cfg.scale)
    res = dict(idx=idx, out=out, lse=lse, n_visible=n_vis)
    if with_scores:
        res["scores"] = scores
    return res


def block_step(inp: dict, pairs: Sequence[tuple]) -> dict:
    """Block-sparse decode for chosen (sequence, head) pairs of a block workload."""
    cfg = inp["cfg"]
    outs, sels, scores = [], [], []
    for b, h in pairs:
        q = _host64(inp["q"][b, h])
        K = _host64(inp["K"][b, :, h])
        V = _host64(inp["V"][b, :, h])
        o, s, bs = block_sparse(q, K, V, cfg.block, cfg.top_blocks, cfg.sink_blocks, cfg.window, cfg.scale)
        outs.append(o); sels.append(s); scores.append(bs)
    return dict(out=np.stack(outs), sel=np.stack(sels), block_scores=np.stack(scores))


def nsa_step(inp: dict, pairs: Sequence[tuple]) -> dict:
    """nsa_decode_group on workload tensors for (sequence b, KV head g) pairs,
    with the compression branch on the stored bf16 cache (nsa_compress):
    q [B, H, D], K and V [B, L, H_kv, D], gates [B, H, 3]; query heads
    g*G .. g*G+G-1 share KV head g (G = H / H_kv).  Returns per pair
    (out [G, D], chosen blocks, p_cmp [G, n_blocks])."""
    cfg = inp["cfg"]
    G = cfg.H // cfg.H_kv
    res = {}
    for b, g in pairs:
        hs = slice(g * G, (g + 1) * G)
        K, V = _host64(inp["K"][b, :, g]), _host64(inp["V"][b, :, g])
        cache = (nsa_compress(K, cfg.block), nsa_compress(V, cfg.block))
        res[(b, g)] = nsa_decode_group(_host64(inp["q"][b, hs]), K, V, cfg.block, cfg.top_blocks, cfg.window,
                                       _host64(inp["gates"][b, hs]), cfg.scale, compressed=cache)
    return res


def csa_step(inp: dict, rows: Sequence[int]) -> dict:
    """The CSA decode of the given sequences from the workload's streams:
    compressed entries (csa_compress; stored as bf16, the indexer keys as
    e4m3), index scores over the n_c compressed keys, Top-K, then csa_attend
    over the chosen entries and the raw window.  Returns out [rows, H, c],
    idx [rows, k], scores [rows, n_c], kv_comp / ki_comp (lists of [n_c, .])."""
    import torch
    cfg = inp["cfg"]
    outs, idxs, scs, kvs, kis = [], [], [], [], []
    for r in rows:
        kv = csa_compress(*(_host64(inp[n][r]) for n in ("Ca", "Cb", "Za", "Zb")), _host64(inp["Ba"]),
                          _host64(inp["Bb"]), cfg.m)
        kv = bf16_round(kv)  # the entries are stored in bf16
        ki = csa_compress(*(_host64(inp[n][r]) for n in ("CIa", "CIb", "ZIa", "ZIb")), _host64(inp["BIa"]),
                          _host64(inp["BIb"]), cfg.m)
        ki = torch.from_numpy(ki).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        sc = index_scores(_host64(inp["q_idx"][r: r + 1]), _host64(inp["w"][r: r + 1]), ki, [0], [cfg.n_c])
        sel = topk(sc, [cfg.n_c], cfg.topk)[0]
        outs.append(csa_attend(_host64(inp["q"][r]), kv, _host64(inp["Ca"][r]), sel, cfg.window, cfg.scale))
        idxs.append(sel)
        scs.append(sc[0])
        kvs.append(kv)
        kis.append(ki)
    return dict(out=np.stack(outs), idx=np.stack(idxs), scores=np.stack(scs), kv_comp=kvs, ki_comp=kis)
