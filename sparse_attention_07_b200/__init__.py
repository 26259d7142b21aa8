"""Thin Python binding of libsparse_attn.so (C ABI in include/sparse_attn.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There
is no CPU or library fallback: if the shared library is missing or a call
fails, an exception is raised.

Functions take torch tensors on the current CUDA device and launch on
``torch.cuda.current_stream()``; outputs are allocated with torch unless given.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparse_attn.so")
_lib = None

SA_OK, SA_EINVAL, SA_EUNSUPPORTED, SA_ECUDA, SA_ETIMEOUT = range(5)
SA_F32, SA_E4M3, SA_BF16 = range(3)

EXPORTS = (
    "sa_status_string", "sa_version", "sa_check_device_error", "sa_index_scores", "sa_topk_select",
    "sa_sparse_mla_workspace_size", "sa_sparse_mla_prefill_workspace_size", "sa_sparse_mla_decode",
    "sa_sparse_mla_prefill",
    "sa_block_mean_pool", "sa_block_sparse_attn", "sa_sparse_mla_decode_static",
    "sa_dense_mla_workspace_size", "sa_dense_mla_decode", "sa_mla_absorb_query", "sa_mla_up_project",
    "sa_nsa_compress", "sa_nsa_decode", "sa_csa_compress", "sa_csa_window_index",
    "sa_index_scores_hist", "sa_topk_select_hist", "sa_set_wait_limit_ns",
    "sa_index_candidates", "sa_topk_from_candidates", "sa_sparse_mla_decode_bf16", "sa_sparse_mla_prefill_bf16",
    "sa_mla_up_project_bf16",
)

# Size of the library's static device array behind sparse_mla_decode_static
# (SA_STATIC_SCRATCH_BYTES in include/sparse_attn.h).
STATIC_SCRATCH_BYTES = (40 << 20) + (256 << 10)


class SparseAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        name = lib().sa_status_string(status).decode()
        super().__init__(f"{fn} returned {name} ({status})")
        self.status = status


def lib():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_attention_07_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.sa_status_string.restype = ctypes.c_char_p
        L.sa_status_string.argtypes = [I]
        L.sa_version.restype = I
        L.sa_check_device_error.argtypes = [ctypes.POINTER(I), P]
        L.sa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.sa_index_scores.argtypes = [P, P, P, I64, I, P, I, P, P, I, I, I, I64, P, P]
        L.sa_topk_select.argtypes = [P, I64, P, I, I, P, P]
        L.sa_index_scores_hist.argtypes = [P, P, P, I64, I, P, I, P, P, I, I, I, I64, P, P, P]
        L.sa_topk_select_hist.argtypes = [P, I64, P, I, I, P, P, P]
        L.sa_index_candidates.argtypes = [P, P, P, I64, I, P, I, P, I, I, I, I, I64, P, P, P, P]
        L.sa_topk_from_candidates.argtypes = [P, I64, P, P, I, I, P, P, P]
        L.sa_sparse_mla_workspace_size.restype = SZ
        L.sa_sparse_mla_workspace_size.argtypes = [I, I, I, I]
        L.sa_sparse_mla_decode.argtypes = [P, P, P, I64, P, I64, I64, P, I, P, P, I, I, I, I, I, F, P, P, P, SZ, P]
        L.sa_sparse_mla_prefill_workspace_size.restype = SZ
        L.sa_sparse_mla_prefill_workspace_size.argtypes = [I, I, I, I]
        L.sa_sparse_mla_prefill.argtypes = [P, P, P, I64, P, I64, I64, P, I, P, P, I, I, I, I, I, F, P, P, P, SZ, P]
        L.sa_sparse_mla_decode_bf16.argtypes = L.sa_sparse_mla_decode.argtypes
        L.sa_sparse_mla_prefill_bf16.argtypes = L.sa_sparse_mla_prefill.argtypes
        L.sa_dense_mla_workspace_size.restype = SZ
        L.sa_dense_mla_workspace_size.argtypes = [I, I, I, I]
        L.sa_dense_mla_decode.argtypes = [P, P, P, I64, P, I64, I64, P, I, P, P, I, I, I, I, I, F, P, P, P, SZ, P]
        L.sa_mla_absorb_query.argtypes = [P, P, I, I, I, I, P, P]
        L.sa_mla_up_project.argtypes = [P, P, I, I, I, I, P, P]
        L.sa_mla_up_project_bf16.argtypes = [P, P, I, I, I, I, P, P]
        L.sa_sparse_mla_decode_static.argtypes = [P, P, P, I64, P, I64, I64, P, I, P, P, I, I, I, I, I, F, P, P, P]
        L.sa_block_mean_pool.argtypes = [P, I64, I64, I64, I, I, I, I, I, P, I64, P]
        L.sa_block_sparse_attn.argtypes = [P, P, I64, P, P, I64, I64, I64, I, I, I, I, I, I, I, I, F, P, P, P]
        L.sa_nsa_compress.argtypes = [P, P, I64, I64, I64, I, I, I, I, I, P, P, I64, P]
        L.sa_nsa_decode.argtypes = [P, P, P, I64, I64, I64, P, P, I64, P, I, I, I, I, I, I, I, I, F, P, P, P]
        L.sa_csa_compress.argtypes = [P, P, P, P, I64, I64, P, P, I, I, I, I, I, I, P, I, I64, I64, P]
        L.sa_csa_window_index.argtypes = [P, I, I, P, I, I, P, P]
        for name in EXPORTS:
            if name not in ("sa_status_string", "sa_version", "sa_sparse_mla_workspace_size",
                            "sa_sparse_mla_prefill_workspace_size", "sa_dense_mla_workspace_size"):
                getattr(L, name).restype = I
        _lib = L
    return _lib


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(fn: str, st: int):
    if st != SA_OK:
        raise SparseAttnError(fn, st)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SA_F32
    if t.dtype == torch.float8_e4m3fn:
        return SA_E4M3
    raise TypeError(f"unsupported indexer dtype {t.dtype}")


def check_device_error() -> int:
    """Synchronise the current stream; return (and clear) the device error word."""
    code = ctypes.c_int(0)
    st = lib().sa_check_device_error(ctypes.byref(code), _stream())
    if st not in (SA_OK, SA_ETIMEOUT):
        raise SparseAttnError("sa_check_device_error", st)
    return code.value


def set_wait_limit_ns(limit_ns: int) -> None:
    """Time limit of the kernels' waits on other parties for the current GPU
    (0: the default of one second).  Synchronous."""
    _check("sa_set_wait_limit_ns", lib().sa_set_wait_limit_ns(int(limit_ns)))


HIST_BINS = 4096


def topk_histogram(rows: int, device) -> torch.Tensor:
    """A zeroed [rows, 4096] int32 buffer for index_scores(hist=...) and
    topk_select(hist=...): the Top-K leaves it zeroed, so one serves every step."""
    return torch.zeros(rows, HIST_BINS, dtype=torch.int32, device=device)


def index_scores(q_idx, w, k_idx_cache, n_visible, pages_per_seq: int, page_table=None, seq_of_row=None,
                 scores=None, scores_ld: Optional[int] = None, hist=None):
    """Lightning-indexer scores [rows, scores_ld] fp32 (entries past n_visible untouched).
    With `hist` (zeroed [rows, 4096] int32) it also counts each row's first
    Top-K digit, for topk_select(hist=...)."""
    rows, H_I, d_I = q_idx.shape
    ld = scores_ld or pages_per_seq * 64
    if scores is None:
        scores = torch.empty(rows, ld, dtype=torch.float32, device=q_idx.device)
    pool_pages = k_idx_cache.shape[0] // 64
    args = (_p(q_idx), _p(w), _p(k_idx_cache), pool_pages, _dtype_code(q_idx), _p(page_table), pages_per_seq,
            _p(seq_of_row), _p(n_visible), rows, H_I, d_I, scores.stride(0), _p(scores))
    if hist is None:
        st = lib().sa_index_scores(*args, _stream())
        _check("sa_index_scores", st)
    else:
        st = lib().sa_index_scores_hist(*args, _p(hist), _stream())
        _check("sa_index_scores_hist", st)
    return scores


def topk_select(scores, n_valid, k: int, idx_out=None, hist=None):
    """Exact Top-K positions [rows, k] int32, ascending, -1 padded.  With
    `hist` (as filled by index_scores(hist=...)) the selection starts from it
    and clears it."""
    rows = scores.shape[0]
    if idx_out is None:
        idx_out = torch.empty(rows, k, dtype=torch.int32, device=scores.device)
    if hist is None:
        st = lib().sa_topk_select(_p(scores), scores.stride(0), _p(n_valid), rows, k, _p(idx_out), _stream())
        _check("sa_topk_select", st)
    else:
        st = lib().sa_topk_select_hist(_p(scores), scores.stride(0), _p(n_valid), rows, k, _p(hist), _p(idx_out),
                                       _stream())
        _check("sa_topk_select_hist", st)
    return idx_out


def candidate_buffers(rows: int, cand_ld: int, device):
    """(cand [rows, cand_ld] uint64 as int64, cand_cnt [rows] int32 zeroed,
    hist [rows, 4096] int32 zeroed) for index_candidates / topk_from_candidates:
    the Top-K leaves the counts zeroed, so one set serves every step."""
    return (torch.empty(rows, cand_ld, dtype=torch.int64, device=device),
            torch.zeros(rows, dtype=torch.int32, device=device),
            torch.zeros(rows, HIST_BINS, dtype=torch.int32, device=device))


def index_candidates(q_idx, w, k_idx_cache, n_visible, pages_per_seq: int, k: int, cand, cand_cnt, hist,
                     page_table=None):
    """Indexer scores of one query row per sequence, kept only where they can
    still be among the row's k largest: cand[r, :cand_cnt[r]] holds
    (order key << 32) | (0xFFFFFFFF - position) (read as int64), and hist
    counts every score's first digit."""
    rows, H_I, d_I = q_idx.shape
    pool_pages = k_idx_cache.shape[0] // 64
    st = lib().sa_index_candidates(_p(q_idx), _p(w), _p(k_idx_cache), pool_pages, _dtype_code(q_idx),
                                   _p(page_table), pages_per_seq, _p(n_visible), rows, H_I, d_I, k,
                                   cand.stride(0), _p(cand), _p(cand_cnt), _p(hist), _stream())
    _check("sa_index_candidates", st)
    return cand


def topk_from_candidates(cand, cand_cnt, n_valid, k: int, hist, idx_out=None):
    """Exact Top-K positions [rows, k] int32 (as topk_select) from the output of
    index_candidates; clears hist and cand_cnt."""
    rows = cand.shape[0]
    if idx_out is None:
        idx_out = torch.empty(rows, k, dtype=torch.int32, device=cand.device)
    st = lib().sa_topk_from_candidates(_p(cand), cand.stride(0), _p(cand_cnt), _p(n_valid), rows, k, _p(hist),
                                       _p(idx_out), _stream())
    _check("sa_topk_from_candidates", st)
    return idx_out


def sparse_mla_workspace_size(rows: int, H: int, k: int, d_c: int = 512) -> int:
    return int(lib().sa_sparse_mla_workspace_size(rows, H, k, d_c))


def _mla_args(q_lat, q_rope, c_cache, kr_cache, idx, out, lse):
    rows, H, d_c = q_lat.shape
    d_R = q_rope.shape[2]
    k = idx.shape[1]
    if out is None:
        out = torch.empty(rows, H, d_c, dtype=torch.float32, device=q_lat.device)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"sparse MLA output must be float32 or bfloat16, not {out.dtype}")
    pool_pages = c_cache.shape[0] // 64
    return rows, H, d_c, d_R, k, out, lse, pool_pages


def sparse_mla_decode(q_lat, q_rope, c_cache, kr_cache, idx, scale: float, pages_per_seq: int, page_table=None,
                      seq_of_row=None, out=None, lse=None, workspace=None):
    """Sparse MLA (latent aggregate) [rows, H, d_c], fp32 (or bf16 when `out`
    is a bf16 tensor); optional lse [rows, H]."""
    rows, H, d_c, d_R, k, out, lse, pool_pages = _mla_args(q_lat, q_rope, c_cache, kr_cache, idx, out, lse)
    need = sparse_mla_workspace_size(rows, H, k, d_c)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_lat.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    name = "sa_sparse_mla_decode_bf16" if out.dtype == torch.bfloat16 else "sa_sparse_mla_decode"
    st = getattr(lib(), name)(_p(q_lat), _p(q_rope), _p(c_cache), c_cache.stride(0), _p(kr_cache),
                              kr_cache.stride(0), pool_pages, _p(page_table), pages_per_seq, _p(seq_of_row),
                              _p(idx), rows, H, k, d_c, d_R, float(scale), _p(out), _p(lse), _p(workspace),
                              wbytes, _stream())
    _check(name, st)
    return out


def sparse_mla_prefill_workspace_size(rows: int, H: int, k: int, d_c: int = 512) -> int:
    return int(lib().sa_sparse_mla_prefill_workspace_size(rows, H, k, d_c))


def sparse_mla_prefill(q_lat, q_rope, c_cache, kr_cache, idx, scale: float, pages_per_seq: int, page_table=None,
                       seq_of_row=None, out=None, lse=None, workspace=None):
    rows, H, d_c, d_R, k, out, lse, pool_pages = _mla_args(q_lat, q_rope, c_cache, kr_cache, idx, out, lse)
    if workspace is None and rows > 0:
        workspace = torch.empty(sparse_mla_prefill_workspace_size(rows, H, k, d_c), dtype=torch.uint8,
                                device=q_lat.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    name = "sa_sparse_mla_prefill_bf16" if out.dtype == torch.bfloat16 else "sa_sparse_mla_prefill"
    st = getattr(lib(), name)(_p(q_lat), _p(q_rope), _p(c_cache), c_cache.stride(0), _p(kr_cache),
                              kr_cache.stride(0), pool_pages, _p(page_table), pages_per_seq, _p(seq_of_row),
                              _p(idx), rows, H, k, d_c, d_R, float(scale), _p(out), _p(lse), _p(workspace),
                              wbytes, _stream())
    _check(name, st)
    return out


def dense_mla_workspace_size(rows: int, H: int, L_max: int, d_c: int = 512) -> int:
    return int(lib().sa_dense_mla_workspace_size(rows, H, L_max, d_c))


def dense_mla_decode(q_lat, q_rope, c_cache, kr_cache, n_visible, L_max: int, scale: float, pages_per_seq: int,
                     page_table=None, seq_of_row=None, out=None, lse=None, workspace=None):
    """Dense MLA over every visible position (the short-sequence mode): row r
    attends to positions 0 .. n_visible[r]-1.  [rows, H, d_c] fp32."""
    rows, H, d_c = q_lat.shape
    d_R = q_rope.shape[2]
    if out is None:
        out = torch.empty(rows, H, d_c, dtype=torch.float32, device=q_lat.device)
    pool_pages = c_cache.shape[0] // 64
    if workspace is None and rows > 0:
        workspace = torch.empty(dense_mla_workspace_size(rows, H, L_max, d_c), dtype=torch.uint8,
                                device=q_lat.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().sa_dense_mla_decode(_p(q_lat), _p(q_rope), _p(c_cache), c_cache.stride(0), _p(kr_cache),
                                   kr_cache.stride(0), pool_pages, _p(page_table), pages_per_seq, _p(seq_of_row),
                                   _p(n_visible), rows, H, L_max, d_c, d_R, float(scale), _p(out), _p(lse),
                                   _p(workspace), wbytes, _stream())
    _check("sa_dense_mla_decode", st)
    return out


def mla_absorb_query(q_c, U_K, q_lat=None):
    """q_lat[r,h,:] = U_K[h]^T q_c[r,h,:]: q_c [rows,H,d_C] bf16, U_K [H,d_C,d_c] bf16 -> [rows,H,d_c] bf16."""
    rows, H, d_C = q_c.shape
    d_c = U_K.shape[2]
    if q_lat is None:
        q_lat = torch.empty(rows, H, d_c, dtype=torch.bfloat16, device=q_c.device)
    _check("sa_mla_absorb_query", lib().sa_mla_absorb_query(_p(q_c), _p(U_K), rows, H, d_C, d_c, _p(q_lat), _stream()))
    return q_lat


def mla_up_project(o_lat, U_V, out=None):
    """out[r,h,:] = U_V[h] o_lat[r,h,:]: o_lat [rows,H,d_c] fp32 or bf16, U_V [H,d_v,d_c] bf16 -> [rows,H,d_v] fp32."""
    rows, H, d_c = o_lat.shape
    d_v = U_V.shape[1]
    if out is None:
        out = torch.empty(rows, H, d_v, dtype=torch.float32, device=o_lat.device)
    if o_lat.dtype == torch.bfloat16:
        name = "sa_mla_up_project_bf16"
    elif o_lat.dtype == torch.float32:
        name = "sa_mla_up_project"
    else:
        raise TypeError(f"o_lat must be float32 or bfloat16, not {o_lat.dtype}")
    _check(name, getattr(lib(), name)(_p(o_lat), _p(U_V), rows, H, d_c, d_v, _p(out), _stream()))
    return out


def sparse_mla_decode_static(q_lat, q_rope, c_cache, kr_cache, idx, scale: float, pages_per_seq: int,
                             page_table=None, seq_of_row=None, out=None, lse=None):
    """sparse_mla_decode without a workspace: for callers that cannot allocate
    device memory, the split-key partial states go to the library's static
    device array (STATIC_SCRATCH_BYTES).  Calls share that array, so calls that
    may overlap on the GPU must be ordered on one stream.  ``out`` and ``lse``
    can be passed in so that the call itself allocates nothing."""
    rows, H, d_c, d_R, k, out, lse, pool_pages = _mla_args(q_lat, q_rope, c_cache, kr_cache, idx, out, lse)
    need = sparse_mla_workspace_size(rows, H, k, d_c)
    if need > STATIC_SCRATCH_BYTES:
        raise ValueError(f"sparse_mla_decode_static: {rows} rows x {H} heads x k={k} need {need} bytes of "
                         f"split-key state, the static array holds {STATIC_SCRATCH_BYTES}; "
                         "use sparse_mla_decode with a workspace")
    st = lib().sa_sparse_mla_decode_static(_p(q_lat), _p(q_rope), _p(c_cache), c_cache.stride(0), _p(kr_cache),
                                           kr_cache.stride(0), pool_pages, _p(page_table), pages_per_seq,
                                           _p(seq_of_row), _p(idx), rows, H, k, d_c, d_R, float(scale), _p(out),
                                           _p(lse), _stream())
    _check("sa_sparse_mla_decode_static", st)
    return out


def block_mean_pool(K, block: int = 64, pooled=None):
    """Mean-pooled complete blocks: K [B, L, H, D] bf16 -> [B, H, L//block, D] fp32."""
    B, L, H, D = K.shape
    nb = L // block
    if pooled is None:
        pooled = torch.empty(B, H, max(nb, 1), D, dtype=torch.float32, device=K.device)
    st = lib().sa_block_mean_pool(_p(K), K.stride(0), K.stride(1), K.stride(2), B, L, H, D, block, _p(pooled),
                                  pooled.shape[2], _stream())
    _check("sa_block_mean_pool", st)
    return pooled


def block_sparse_attn(q, pooled, K, V, block: int, top_blocks: int, sink_blocks: int, window: int, scale: float,
                      out=None, sel_blocks=None):
    """Block-sparse decode of the query at position L-1: out [B, H, D] fp32."""
    B, L, H, D = K.shape
    if out is None:
        out = torch.empty(B, H, D, dtype=torch.float32, device=q.device)
    st = lib().sa_block_sparse_attn(_p(q), _p(pooled), pooled.shape[2], _p(K), _p(V), K.stride(0), K.stride(1),
                                    K.stride(2), B, H, D, L, block, top_blocks, sink_blocks, window, float(scale),
                                    _p(out), _p(sel_blocks), _stream())
    _check("sa_block_sparse_attn", st)
    return out


def nsa_compress(K, V, block: int = 64, Kc=None, Vc=None):
    """NSA compressed cache: bf16 block means of K and V [B, L, H_kv, D] ->
    Kc, Vc [B, H_kv, L//block, D] bf16 (complete blocks only)."""
    B, L, Hkv, D = K.shape
    nb = L // block
    if Kc is None:
        Kc = torch.empty(B, Hkv, max(nb, 1), D, dtype=torch.bfloat16, device=K.device)
    if Vc is None:
        Vc = torch.empty_like(Kc)
    if V.stride() != K.stride() or not (Kc.is_contiguous() and Vc.is_contiguous()):
        raise ValueError("K and V must share one layout; Kc and Vc must be contiguous")
    st = lib().sa_nsa_compress(_p(K), _p(V), K.stride(0), K.stride(1), K.stride(2), B, L, Hkv, D, block, _p(Kc),
                               _p(Vc), Kc.shape[2], _stream())
    _check("sa_nsa_compress", st)
    return Kc, Vc


def nsa_decode(q, K, V, Kc, Vc, gates, block: int, top_blocks: int, window: int, scale: float, out=None,
               sel_blocks=None):
    """NSA three-branch decode of the query at position L-1 of every head:
    q [B, H, D] bf16, K and V [B, L, H_kv, D] bf16, Kc and Vc from
    nsa_compress, gates [B, H, 3] fp32 -> out [B, H, D] fp32."""
    B, L, Hkv, D = K.shape
    H = q.shape[1]
    if V.stride() != K.stride() or not (Kc.is_contiguous() and Vc.is_contiguous()):
        raise ValueError("K and V must share one layout; Kc and Vc must be contiguous")
    if out is None:
        out = torch.empty(B, H, D, dtype=torch.float32, device=q.device)
    st = lib().sa_nsa_decode(_p(q), _p(K), _p(V), K.stride(0), K.stride(1), K.stride(2), _p(Kc), _p(Vc),
                             Kc.shape[2], _p(gates), B, H, Hkv, D, L, block,
                             top_blocks, window, float(scale), _p(out), _p(sel_blocks), _stream())
    _check("sa_nsa_decode", st)
    return out


def csa_compress(Ca, Cb, Za, Zb, Ba, Bb, m: int, out, out_seq_stride: int, out_row_stride: int, g0: int = 0,
                 g1: Optional[int] = None):
    """CSA compressed entries g0 .. g1-1 of every sequence: streams [S, L, c]
    bf16 (one layout for all four), biases [m, c] fp32; written into `out`
    (bf16 or e4m3) at s*out_seq_stride + g*out_row_stride (elements)."""
    S, L, c = Ca.shape
    if not (Cb.stride() == Za.stride() == Zb.stride() == Ca.stride()):
        raise ValueError("the four streams must share one layout")
    g1 = L // m if g1 is None else g1
    code = 1 if out.dtype == torch.float8_e4m3fn else (2 if out.dtype == torch.bfloat16 else -1)
    st = lib().sa_csa_compress(_p(Ca), _p(Cb), _p(Za), _p(Zb), Ca.stride(0), Ca.stride(1), _p(Ba), _p(Bb), S, L, m,
                               c, g0, g1, _p(out), code, out_seq_stride, out_row_stride, _stream())
    _check("sa_csa_compress", st)
    return out


def csa_window_index(topk_idx, raw_len, window: int, win_base: int, idx_out=None):
    """[rows, k + window] int32: the selected entries, then the window slots."""
    rows, k = topk_idx.shape
    if idx_out is None:
        idx_out = torch.empty(rows, k + window, dtype=torch.int32, device=topk_idx.device)
    st = lib().sa_csa_window_index(_p(topk_idx), rows, k, _p(raw_len), window, win_base, _p(idx_out), _stream())
    _check("sa_csa_window_index", st)
    return idx_out
