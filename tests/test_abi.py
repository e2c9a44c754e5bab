"""The C-ABI library loads, exports every entry point include/bi.h declares,
and rejects bad arguments on the host before touching the GPU. No GPU needed:
every call here fails (or returns early) before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bi.h")


@pytest.fixture(scope="module")
def bi():
    from invariant_deterministic_03_b200 import build
    build.build()
    from invariant_deterministic_03_b200 import bi as mod
    return mod


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bi_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ["bi_rmsnorm", "bi_gemm", "bi_kv_append", "bi_attn_decode", "bi_attn_prefill",
                 "bi_attn_workspace_size", "bi_forward", "bi_model_create", "bi_last_error"]:
        assert want in names


def test_library_exports_every_declared_symbol(bi):
    for name in _declared():
        assert hasattr(bi.lib, name), f"libbi.so does not export {name}"
    assert set(bi.EXPORTS) >= set(_declared())


def _st(bi, fn, *args):
    return getattr(bi.lib, fn)(*args)


def test_rmsnorm_host_checks(bi):
    p = 0x1000  # aligned fake pointer; never dereferenced on these paths
    assert _st(bi, "bi_rmsnorm", None, p, p, 4, 512, 1e-6, None) == bi.BI_ERR_INVALID_ARG
    assert _st(bi, "bi_rmsnorm", p, p, p, 4, 500, 1e-6, None) == bi.BI_ERR_SHAPE
    assert _st(bi, "bi_rmsnorm", p, p, p, 4, 65536, 1e-6, None) == bi.BI_ERR_SHAPE
    assert _st(bi, "bi_rmsnorm", p + 2, p, p, 4, 512, 1e-6, None) == bi.BI_ERR_ALIGN
    assert _st(bi, "bi_rmsnorm", p, p, p, -1, 512, 1e-6, None) == bi.BI_ERR_INVALID_ARG
    assert _st(bi, "bi_rmsnorm", p, p, p, 0, 512, 1e-6, None) == bi.BI_OK  # empty batch: no-op


def test_gemm_host_checks(bi):
    p = 0x1000
    g = bi.lib.bi_gemm
    assert g(p, 64, p, 64, p, 64, bi.BI_BF16, 4, 64, 63, None) == bi.BI_ERR_SHAPE      # K % 8
    assert b"multiple" in bi.lib.bi_last_error()
    assert g(p, 64, p, 64, p, 64, bi.BI_BF16, 4, 60, 64, None) == bi.BI_ERR_SHAPE      # N % 8
    assert g(p, 60, p, 64, p, 64, bi.BI_BF16, 4, 64, 64, None) == bi.BI_ERR_SHAPE      # lda < K
    assert g(p, 72, p, 68, p, 64, bi.BI_BF16, 4, 64, 64, None) == bi.BI_ERR_ALIGN      # ldw % 8
    assert g(p + 8, 64, p, 64, p, 64, bi.BI_BF16, 4, 64, 64, None) == bi.BI_ERR_ALIGN  # A align
    assert g(p, 64, p, 64, p, 64, 7, 4, 64, 64, None) == bi.BI_ERR_INVALID_ARG         # dtype
    assert g(None, 64, p, 64, p, 64, bi.BI_BF16, 4, 64, 64, None) == bi.BI_ERR_INVALID_ARG
    assert g(p, 64, p, 64, p, 64, bi.BI_BF16, 0, 64, 64, None) == bi.BI_OK             # M == 0
    assert g(p, 64, p, 64, p, 64, bi.BI_F32, 5, 0, 64, None) == bi.BI_OK               # N == 0


def test_attention_host_checks(bi):
    p = 0x1000
    sh = bi.attn_shape(32, 8, 100, 10, 160)
    n = ctypes.c_size_t(0)
    assert bi.lib.bi_attn_workspace_size(ctypes.byref(sh), 7, ctypes.byref(n)) == bi.BI_OK
    # 7 tokens x 32 heads x ceil(160/512)=1 split x (128 + 2) floats, rounded
    # up to 256 bytes, then the 256-byte work counter
    assert n.value == 7 * 32 * 1 * 130 * 4 + 256
    sh_big = bi.attn_shape(32, 8, 100, 10, 8192)
    assert bi.lib.bi_attn_workspace_size(ctypes.byref(sh_big), 32, ctypes.byref(n)) == bi.BI_OK
    assert n.value == 32 * 32 * 16 * 130 * 4 + 256
    bad = bi.attn_shape(32, 6, 100, 10, 160)   # 32 % 6 != 0
    assert bi.lib.bi_attn_workspace_size(ctypes.byref(bad), 1, ctypes.byref(n)) == bi.BI_ERR_SHAPE
    g3 = bi.attn_shape(48, 16, 100, 10, 160)   # 3 q heads per kv head unsupported
    assert bi.lib.bi_attn_workspace_size(ctypes.byref(g3), 1, ctypes.byref(n)) == bi.BI_ERR_SHAPE
    hd = bi.attn_shape(32, 8, 100, 10, 160)
    hd.head_dim = 64
    assert bi.lib.bi_attn_workspace_size(ctypes.byref(hd), 1, ctypes.byref(n)) == bi.BI_ERR_SHAPE
    dec = bi.lib.bi_attn_decode
    # workspace too small
    assert dec(p, 4096, p, p, p, p, 4, ctypes.byref(sh), p, 4096, p, 16, None) == bi.BI_ERR_WORKSPACE
    # ldq too small
    assert dec(p, 2048, p, p, p, p, 4, ctypes.byref(sh), p, 4096, p, 1 << 30, None) == bi.BI_ERR_SHAPE
    # empty batch is a no-op
    assert dec(p, 4096, p, p, p, p, 0, ctypes.byref(sh), p, 4096, p, 0, None) == bi.BI_OK
    pre = bi.lib.bi_attn_prefill
    assert pre(p, 4096, None, 8, 8, p, p, p, p, 1, ctypes.byref(sh), p, 4096, p, 1 << 30, None) == bi.BI_ERR_INVALID_ARG


def test_kv_append_and_pointwise_host_checks(bi):
    p = 0x1000
    kv = bi.KVLayout(10, 8, 128, 16)
    assert bi.lib.bi_kv_append(p, p, 512, p, 3, p, p, ctypes.byref(kv), None) == bi.BI_ERR_SHAPE
    kv_bad = bi.KVLayout(10, 8, 128, 32)
    assert bi.lib.bi_kv_append(p, p, 1024, p, 3, p, p, ctypes.byref(kv_bad), None) == bi.BI_ERR_SHAPE
    assert bi.lib.bi_kv_append(p, p, 1024, p, 0, p, p, ctypes.byref(kv), None) == bi.BI_OK
    assert bi.lib.bi_embed(p, 4, p, 100, 12, p, None) == bi.BI_ERR_ALIGN
    assert bi.lib.bi_argmax(p, 2, 10, 5, p, None) == bi.BI_ERR_INVALID_ARG
    assert bi.lib.bi_swiglu(p, 0, 64, p, None) == bi.BI_OK
    assert bi.lib.bi_rope(p, 64, 1, p, 1, p, 16, None) == bi.BI_ERR_SHAPE


def test_model_create_checks(bi):
    cfg = bi.ModelConfig(2, 4096, 32, 8, 14336, 32000, 4096, 1e-6, 1e4)
    w = bi.ModelWeights(*([0x1000] * 9))
    h = ctypes.c_void_p(0)
    assert bi.lib.bi_model_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == bi.BI_OK
    n = ctypes.c_size_t(0)
    assert bi.lib.bi_forward_workspace_size(h, 16, 4, 4096, ctypes.byref(n)) == bi.BI_OK
    assert n.value > 16 * 4096 * 4
    bi.lib.bi_model_destroy(h)
    bad = bi.ModelConfig(2, 4000, 32, 8, 14336, 32000, 4096, 1e-6, 1e4)
    assert bi.lib.bi_model_create(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == bi.BI_ERR_SHAPE


def test_gemm_epilogue_host_checks(bi):
    p = 0x1000
    g = bi.lib.bi_gemm
    assert g(p, 64, p, 64, p, 64, bi.BI_F32_ADD, 4, 64, 60, None) == bi.BI_ERR_SHAPE   # K % 8
    sw = bi.lib.bi_gemm_swiglu
    assert sw(p, 64, p, 64, p, 60, 4, 60, 64, None) == bi.BI_ERR_SHAPE    # F % 8
    assert sw(p, 64, p, 64, p, 8, 4, 16, 64, None) == bi.BI_ERR_SHAPE     # ldo < F
    assert sw(None, 64, p, 64, p, 16, 4, 16, 64, None) == bi.BI_ERR_INVALID_ARG
    assert sw(p, 64, p, 64, p, 16, 0, 16, 64, None) == bi.BI_OK           # M == 0: nothing to do


def test_wait_bound_check_host_checks(bi):
    assert bi.lib.bi_check_wait_bound(999, None) == bi.BI_ERR_INVALID_ARG
    assert bi.lib.bi_check_wait_bound((1 << 32) + 1, None) == bi.BI_ERR_INVALID_ARG
    assert b"limit" in bi.lib.bi_last_error()


def test_gemm_qkv_host_checks(bi):
    p = 0x1000
    g = bi.lib.bi_gemm_qkv
    ok = dict(A=p, lda=512, W=p, ldw=512, qkv=p, ldq=1024, M=4, K=512, hq=4, hkv=2, pos=p, cs=p,
              max_pos=64, slots=p, kc=p, vc=p, pages=8, s=None)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["A"], a["lda"], a["W"], a["ldw"], a["qkv"], a["ldq"], a["M"], a["K"], a["hq"], a["hkv"],
                 a["pos"], a["cs"], a["max_pos"], a["slots"], a["kc"], a["vc"], a["pages"], a["s"])
    assert call(hq=0) == bi.BI_ERR_INVALID_ARG
    assert call(ldq=512) == bi.BI_ERR_SHAPE            # ldq < (4 + 2 * 2) * 128
    assert call(K=500, lda=504, ldw=504) == bi.BI_ERR_SHAPE   # K % 8
    assert call(slots=None) == bi.BI_ERR_INVALID_ARG
    assert call(max_pos=0) == bi.BI_ERR_INVALID_ARG
    assert call(kc=p + 8) == bi.BI_ERR_ALIGN
    assert call(M=0) == bi.BI_OK                        # nothing to do


def test_gemm_rmsnorm_host_checks(bi):
    p = 0x1000
    n = ctypes.c_size_t(0)
    assert bi.lib.bi_gemm_rmsnorm_workspace_size(64, 4096, ctypes.byref(n)) == bi.BI_OK
    assert n.value == 256 + 64 * 4096 * 2                   # row scales (256-byte rounded), then normed rows
    assert bi.lib.bi_gemm_rmsnorm_workspace_size(-1, 8, ctypes.byref(n)) == bi.BI_ERR_INVALID_ARG
    g = bi.lib.bi_gemm_rmsnorm
    ok = dict(x=p, gamma=p, eps=1e-6, W=p, ldw=512, C=p, ldc=256, c=bi.BI_BF16, M=4, N=256, K=512, ws=p,
              wsb=1 << 20, s=None)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["x"], a["gamma"], a["eps"], a["W"], a["ldw"], a["C"], a["ldc"], a["c"], a["M"], a["N"], a["K"],
                 a["ws"], a["wsb"], a["s"])
    assert call(x=None) == bi.BI_ERR_INVALID_ARG
    assert call(ws=None) == bi.BI_ERR_INVALID_ARG
    assert call(c=bi.BI_F32_ADD) == bi.BI_ERR_INVALID_ARG   # no accumulation into C
    assert call(K=500, ldw=504) == bi.BI_ERR_SHAPE           # K % 8
    assert call(gamma=p + 8) == bi.BI_ERR_ALIGN
    assert call(eps=-1.0) == bi.BI_ERR_INVALID_ARG
    assert call(wsb=100) == bi.BI_ERR_WORKSPACE
    assert call(M=0) == bi.BI_OK                            # nothing to do
    sw = bi.lib.bi_gemm_rmsnorm_swiglu
    assert sw(p, p, 1e-6, p, 512, p, 256, 4, 256, 512, p, 100, None) == bi.BI_ERR_WORKSPACE
    assert sw(p, p, 1e-6, p, 512, p, 256, 0, 256, 512, p, 1 << 20, None) == bi.BI_OK
