"""C-ABI checks that need no GPU: the library loads, exports every function
include/sparse_attn.h declares, and rejects bad arguments on the host before
launching anything (no pointer is dereferenced, no CUDA call is made)."""
import ctypes
import os
import re

import pytest

import sparse_attention_07_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_attn.h")

FAKE = ctypes.c_void_p(0x1000)      # 16-byte aligned, never dereferenced on these paths
MISALIGNED = ctypes.c_void_p(0x1004)


@pytest.fixture(scope="module")
def L():
    from sparse_attention_07_b200 import build
    build.build()
    return sa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ("sa_index_scores", "sa_topk_select", "sa_sparse_mla_decode", "sa_sparse_mla_prefill",
              "sa_block_sparse_attn", "sa_block_mean_pool"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert set(declared_functions()) <= set(sa.EXPORTS)


def test_version_and_status_strings(L):
    assert L.sa_version() == 100
    assert L.sa_status_string(sa.SA_EINVAL) == b"SA_EINVAL"
    assert L.sa_status_string(sa.SA_ETIMEOUT) == b"SA_ETIMEOUT"


def test_index_scores_validation(L):
    f = L.sa_index_scores
    good = dict(q=FAKE, w=FAKE, k=FAKE, pool=4, dt=sa.SA_E4M3, pt=None, pps=4, sor=None, nv=FAKE,
                rows=2, H_I=64, d_I=128, ld=256, out=FAKE)

    def call(**kw):
        a = {**good, **kw}
        return f(a["q"], a["w"], a["k"], a["pool"], a["dt"], a["pt"], a["pps"], a["sor"], a["nv"], a["rows"],
                 a["H_I"], a["d_I"], a["ld"], a["out"], None)

    assert call(rows=0) == sa.SA_OK                 # nothing to do, nothing launched
    assert call(rows=-1) == sa.SA_EINVAL
    assert call(H_I=0) == sa.SA_EINVAL
    assert call(pps=0) == sa.SA_EINVAL
    assert call(pool=0) == sa.SA_EINVAL
    assert call(q=None) == sa.SA_EINVAL
    assert call(nv=None) == sa.SA_EINVAL
    assert call(q=MISALIGNED) == sa.SA_EINVAL
    assert call(dt=sa.SA_BF16) == sa.SA_EUNSUPPORTED
    assert call(dt=sa.SA_F32, d_I=130) == sa.SA_EUNSUPPORTED   # not a multiple of 4
    assert call(dt=sa.SA_F32, H_I=65) == sa.SA_EUNSUPPORTED
    assert call(pool=(1 << 27)) == sa.SA_EUNSUPPORTED           # pool rows beyond a tensor map's reach


def test_topk_validation(L):
    f = L.sa_topk_select
    assert f(FAKE, 1024, FAKE, 0, 8, FAKE, None) == sa.SA_OK
    assert f(FAKE, 1024, FAKE, 2, 0, FAKE, None) == sa.SA_EINVAL
    assert f(FAKE, 1024, FAKE, -1, 8, FAKE, None) == sa.SA_EINVAL
    assert f(None, 1024, FAKE, 2, 8, FAKE, None) == sa.SA_EINVAL
    assert f(FAKE, 1022, FAKE, 2, 8, FAKE, None) == sa.SA_EINVAL          # row stride not 16-byte aligned
    assert f(MISALIGNED, 1024, FAKE, 2, 8, FAKE, None) == sa.SA_EINVAL
    assert f(FAKE, 262148, FAKE, 2, 8, FAKE, None) == sa.SA_EUNSUPPORTED  # row longer than the cluster holds


def _mla(L, fn, **kw):
    a = dict(ql=FAKE, qr=FAKE, c=FAKE, cld=512, kr=FAKE, krld=64, pool=4, pt=None, pps=4, sor=None, idx=FAKE,
             rows=2, H=128, k=2048, dc=512, dR=64, scale=0.07, out=FAKE, lse=None)
    a.update(kw)
    args = [a["ql"], a["qr"], a["c"], a["cld"], a["kr"], a["krld"], a["pool"], a["pt"], a["pps"], a["sor"],
            a["idx"], a["rows"], a["H"], a["k"], a["dc"], a["dR"], a["scale"], a["out"], a["lse"]]
    return getattr(L, f"sa_sparse_mla_{fn}")(*args, None, 0, None)


@pytest.mark.parametrize("fn", ["decode", "prefill", "decode_bf16", "prefill_bf16"])
def test_sparse_mla_validation(L, fn):
    assert _mla(L, fn, rows=0) == sa.SA_OK
    assert _mla(L, fn, k=0) == sa.SA_EINVAL
    assert _mla(L, fn, H=0) == sa.SA_EINVAL
    assert _mla(L, fn, idx=None) == sa.SA_EINVAL
    assert _mla(L, fn, scale=float("nan")) == sa.SA_EINVAL
    assert _mla(L, fn, dc=256) == sa.SA_EUNSUPPORTED
    assert _mla(L, fn, dR=32) == sa.SA_EUNSUPPORTED
    assert _mla(L, fn, H=129) == sa.SA_EUNSUPPORTED
    assert _mla(L, fn, cld=520 + 4) == sa.SA_EINVAL            # row stride not 16-byte aligned
    assert _mla(L, fn, c=MISALIGNED) == sa.SA_EINVAL
    assert _mla(L, fn, cld=256) == sa.SA_EINVAL                # stride shorter than a row
    assert _mla(L, fn) == sa.SA_EINVAL                         # no workspace


def test_block_validation(L):
    f = L.sa_block_sparse_attn
    args = dict(q=FAKE, pooled=FAKE, pld=2048, K=FAKE, V=FAKE, sb=8, st=8, sh=128, B=2, H=4, D=128, L=131072,
                block=64, top=16, sink=1, win=512, scale=0.088, out=FAKE, sel=None)

    def call(**kw):
        a = {**args, **kw}
        return f(a["q"], a["pooled"], a["pld"], a["K"], a["V"], a["sb"], a["st"], a["sh"], a["B"], a["H"], a["D"],
                 a["L"], a["block"], a["top"], a["sink"], a["win"], a["scale"], a["out"], a["sel"], None)

    assert call(B=0) == sa.SA_OK
    assert call(D=64) == sa.SA_EUNSUPPORTED
    assert call(block=128) == sa.SA_EUNSUPPORTED
    assert call(top=65) == sa.SA_EUNSUPPORTED
    assert call(L=64 * 4097) == sa.SA_EUNSUPPORTED
    assert call(top=-1) == sa.SA_EINVAL
    assert call(pld=100) == sa.SA_EINVAL
    assert call(st=6) == sa.SA_EINVAL
    assert call(K=None) == sa.SA_EINVAL
    g = L.sa_block_mean_pool
    assert g(FAKE, 8, 8, 128, 2, 1000, 4, 64, 64, FAKE, 15, None) == sa.SA_EUNSUPPORTED
    assert g(FAKE, 8, 8, 128, 2, 1000, 4, 128, 64, FAKE, 10, None) == sa.SA_EINVAL   # pooled too short
    assert g(FAKE, 8, 8, 128, 2, 1000, 4, 128, 0, FAKE, 15, None) == sa.SA_EINVAL


def test_nsa_validation(L):
    f = L.sa_nsa_decode
    args = dict(q=FAKE, K=FAKE, V=FAKE, sb=8 * 131072 * 4 * 128, st=4 * 128, sh=128, Kc=FAKE, Vc=FAKE, cld=2048,
                gates=FAKE, B=8, H=32, Hkv=4, D=128, L=131072, block=64, top=16, win=512, scale=0.088, out=FAKE,
                sel=None)

    def call(**kw):
        a = {**args, **kw}
        return f(a["q"], a["K"], a["V"], a["sb"], a["st"], a["sh"], a["Kc"], a["Vc"], a["cld"], a["gates"], a["B"],
                 a["H"], a["Hkv"], a["D"], a["L"], a["block"], a["top"], a["win"], a["scale"], a["out"], a["sel"],
                 None)

    assert call(B=0) == sa.SA_OK
    assert call(D=64) == sa.SA_EUNSUPPORTED
    assert call(H=34, Hkv=2) == sa.SA_EUNSUPPORTED      # groups of 17 heads
    assert call(block=48) == sa.SA_EUNSUPPORTED
    assert call(top=65) == sa.SA_EUNSUPPORTED
    assert call(win=4097) == sa.SA_EUNSUPPORTED
    assert call(L=64 * 4097) == sa.SA_EUNSUPPORTED
    assert call(H=30) == sa.SA_EINVAL                   # not a whole number of groups
    assert call(L=0) == sa.SA_EINVAL
    assert call(top=-1) == sa.SA_EINVAL
    assert call(cld=100) == sa.SA_EINVAL
    assert call(st=4 * 128 + 4) == sa.SA_EINVAL          # rows not 16-byte aligned
    assert call(q=MISALIGNED) == sa.SA_EINVAL
    assert call(Kc=None) == sa.SA_EINVAL
    assert call(gates=None) == sa.SA_EINVAL
    assert call(scale=float("nan")) == sa.SA_EINVAL
    g = L.sa_nsa_compress
    assert g(FAKE, FAKE, 8, 8, 128, 2, 1000, 4, 64, 64, FAKE, FAKE, 15, None) == sa.SA_EUNSUPPORTED
    assert g(FAKE, FAKE, 8, 8, 128, 2, 1000, 4, 128, 64, FAKE, FAKE, 10, None) == sa.SA_EINVAL   # cache too short
    assert g(FAKE, None, 8, 8, 128, 2, 1000, 4, 128, 64, FAKE, FAKE, 15, None) == sa.SA_EINVAL
    assert g(FAKE, FAKE, 8, 8, 128, 2, 63, 4, 128, 64, None, None, 0, None) == sa.SA_OK       # no complete block


def test_csa_validation(L):
    f = L.sa_csa_compress
    args = dict(Ca=FAKE, Cb=FAKE, Za=FAKE, Zb=FAKE, ss=1024 * 512, rs=512, Ba=FAKE, Bb=FAKE, S=2, L=1024, m=4, c=512,
                g0=0, g1=256, out=FAKE, dt=sa.SA_BF16, oss=256 * 512, ors=512)

    def call(**kw):
        a = {**args, **kw}
        return f(a["Ca"], a["Cb"], a["Za"], a["Zb"], a["ss"], a["rs"], a["Ba"], a["Bb"], a["S"], a["L"], a["m"],
                 a["c"], a["g0"], a["g1"], a["out"], a["dt"], a["oss"], a["ors"], None)

    assert call(S=0) == sa.SA_OK
    assert call(g0=5, g1=5) == sa.SA_OK
    assert call(g1=257) == sa.SA_EINVAL                 # past the complete groups
    assert call(g0=-1) == sa.SA_EINVAL
    assert call(m=0) == sa.SA_EINVAL
    assert call(c=510) == sa.SA_EUNSUPPORTED
    assert call(dt=sa.SA_F32) == sa.SA_EUNSUPPORTED
    assert call(rs=256) == sa.SA_EINVAL                 # rows overlap
    assert call(Za=None) == sa.SA_EINVAL
    assert call(Ba=MISALIGNED) == sa.SA_EINVAL
    assert call(ors=514) == sa.SA_EINVAL
    g = L.sa_csa_window_index
    assert g(FAKE, 0, 16, FAKE, 8, 64, FAKE, None) == sa.SA_OK
    assert g(FAKE, 2, 0, FAKE, 0, 64, FAKE, None) == sa.SA_EINVAL     # no slot at all
    assert g(None, 2, 16, FAKE, 8, 64, FAKE, None) == sa.SA_EINVAL
    assert g(FAKE, 2, 16, FAKE, -1, 64, FAKE, None) == sa.SA_EINVAL
    assert g(FAKE, 2, 16, None, 8, 64, FAKE, None) == sa.SA_EINVAL


def test_check_device_error_rejects_null(L):
    assert L.sa_check_device_error(None, None) == sa.SA_EINVAL


def test_static_scratch_size_matches_the_header():
    """The binding's copy of SA_STATIC_SCRATCH_BYTES (used for its host-side
    check) equals the header's definition."""
    import re
    hdr = open(os.path.join(ROOT, "include", "sparse_attn.h")).read()
    m = re.search(r"#define SA_STATIC_SCRATCH_BYTES \((.*)\)\n", hdr)
    assert m, "definition not found"
    expr = m.group(1).replace("(size_t)", "")
    assert eval(expr, {}) == sa.STATIC_SCRATCH_BYTES


def test_candidate_path_validation(L):
    """sa_index_candidates / sa_topk_from_candidates: bad counts, missing or
    misaligned buffers, a candidate row shorter than the page table's reach,
    and shapes off the tensor-core indexer are refused on the host."""
    f = L.sa_index_candidates
    good = dict(q=FAKE, w=FAKE, k=FAKE, pool=4, dt=sa.SA_E4M3, pt=None, pps=4, nv=FAKE, rows=2, H_I=64, d_I=128,
                topk=64, ld=256, cand=FAKE, cnt=FAKE, hist=FAKE)

    def call(**kw):
        a = {**good, **kw}
        return f(a["q"], a["w"], a["k"], a["pool"], a["dt"], a["pt"], a["pps"], a["nv"], a["rows"], a["H_I"],
                 a["d_I"], a["topk"], a["ld"], a["cand"], a["cnt"], a["hist"], None)

    assert call(rows=0) == sa.SA_OK
    assert call(rows=-1) == sa.SA_EINVAL
    assert call(topk=0) == sa.SA_EINVAL
    assert call(ld=255) == sa.SA_EINVAL                 # shorter than pages_per_seq * 64
    assert call(cand=None) == sa.SA_EINVAL
    assert call(cnt=None) == sa.SA_EINVAL
    assert call(hist=None) == sa.SA_EINVAL
    assert call(hist=MISALIGNED) == sa.SA_EINVAL        # the bound is read in 16-byte pieces
    assert call(q=MISALIGNED) == sa.SA_EINVAL
    assert call(dt=sa.SA_F32) == sa.SA_EUNSUPPORTED     # the tensor-core indexer only
    assert call(d_I=64) == sa.SA_EUNSUPPORTED
    assert call(rows=4097) == sa.SA_EUNSUPPORTED
    assert call(pps=4097, ld=4097 * 64) == sa.SA_EUNSUPPORTED  # rows longer than the Top-K's bitmaps

    g = L.sa_topk_from_candidates
    assert g(FAKE, 256, FAKE, FAKE, 0, 8, FAKE, FAKE, None) == sa.SA_OK
    assert g(FAKE, 256, FAKE, FAKE, -1, 8, FAKE, FAKE, None) == sa.SA_EINVAL
    assert g(FAKE, 256, FAKE, FAKE, 2, 0, FAKE, FAKE, None) == sa.SA_EINVAL
    assert g(FAKE, 0, FAKE, FAKE, 2, 8, FAKE, FAKE, None) == sa.SA_EINVAL
    assert g(None, 256, FAKE, FAKE, 2, 8, FAKE, FAKE, None) == sa.SA_EINVAL
    assert g(FAKE, 256, FAKE, FAKE, 2, 8, None, FAKE, None) == sa.SA_EINVAL
    assert g(ctypes.c_void_p(0x1004), 256, FAKE, FAKE, 2, 8, FAKE, FAKE, None) == sa.SA_EINVAL
    assert g(FAKE, 262144 + 64, FAKE, FAKE, 2, 8, FAKE, FAKE, None) == sa.SA_EUNSUPPORTED


@pytest.mark.parametrize("name", ["sa_mla_up_project", "sa_mla_up_project_bf16"])
def test_up_project_validation(L, name):
    f = getattr(L, name)
    assert f(FAKE, FAKE, 0, 8, 512, 128, FAKE, None) == sa.SA_OK
    assert f(FAKE, FAKE, -1, 8, 512, 128, FAKE, None) == sa.SA_EINVAL
    assert f(None, FAKE, 2, 8, 512, 128, FAKE, None) == sa.SA_EINVAL
    assert f(MISALIGNED, FAKE, 2, 8, 512, 128, FAKE, None) == sa.SA_EINVAL
    assert f(FAKE, FAKE, 2, 8, 500, 128, FAKE, None) == sa.SA_EUNSUPPORTED   # d_c not a multiple of 64
    assert f(FAKE, FAKE, 2, 8, 512, 100, FAKE, None) == sa.SA_EUNSUPPORTED   # d_v not a multiple of 128
