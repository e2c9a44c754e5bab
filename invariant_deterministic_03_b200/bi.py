"""Thin ctypes binding of libbi (include/bi.h) for torch tensors.

Argument marshalling only: every entry point takes device tensors, passes
their data pointers, sizes and the current CUDA stream to the C ABI and raises
:class:`BIError` on a non-zero status. No arithmetic of the path runs here and
there is no CPU fallback: importing this module fails loudly when libbi.so is
missing, and every call fails on a non-B200 device.

The functions named ``bi_*`` mirror the C entry points (outputs passed in);
the short names (``rmsnorm``, ``gemm``, ...) allocate their outputs with torch
and call the same entry points.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbi.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libbi.so is not built ({LIB_PATH}); run "
                      "`python -m invariant_deterministic_03_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

BI_OK, BI_ERR_INVALID_ARG, BI_ERR_SHAPE, BI_ERR_ALIGN, BI_ERR_WORKSPACE, \
    BI_ERR_UNSUPPORTED, BI_ERR_CUDA, BI_ERR_DEVICE_CHECK = range(8)
BI_BF16, BI_F32, BI_F32_ADD = 0, 1, 2
BI_PREC_BF16, BI_PREC_F32, BI_PREC_BF16_MLP, BI_PREC_F16 = 0, 1, 2, 3
PRECISIONS = {"bf16": BI_PREC_BF16, "f32": BI_PREC_F32, "bf16_mlp": BI_PREC_BF16_MLP, "f16": BI_PREC_F16}
HEAD_DIM, PAGE_SIZE, ATTN_TILE, ATTN_SPLIT = 128, 16, 128, 512
GEMM_BM, GEMM_BN, GEMM_BK = 256, 256, 64

_p, _i32, _i64, _f32, _f64, _sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                   ctypes.c_float, ctypes.c_double, ctypes.c_size_t)


class KVLayout(ctypes.Structure):
    _fields_ = [("num_pages", _i32), ("num_kv_heads", _i32), ("head_dim", _i32),
                ("page_size", _i32)]


class AttnShape(ctypes.Structure):
    _fields_ = [("num_q_heads", _i32), ("num_kv_heads", _i32), ("head_dim", _i32),
                ("page_size", _i32), ("num_pages", _i32), ("max_pages_per_seq", _i32),
                ("max_kv_len", _i32), ("scale", _f32)]


class ModelConfig(ctypes.Structure):
    _fields_ = [("n_layers", _i32), ("d_model", _i32), ("n_q_heads", _i32),
                ("n_kv_heads", _i32), ("d_ff", _i32), ("vocab", _i32), ("max_pos", _i32),
                ("rms_eps", _f32), ("rope_theta", _f64), ("precision", _i32)]


class ModelWeights(ctypes.Structure):
    _fields_ = [(n, _p) for n in ("embed", "attn_norm", "w_qkv", "w_o", "mlp_norm",
                                  "w_gate_up", "w_down", "final_norm", "lm_head")]


class Batch(ctypes.Structure):
    _fields_ = [("tokens", _p), ("positions", _p), ("slot_mapping", _p), ("cu_q", _p),
                ("seq_lens", _p), ("block_table", _p), ("logits_rows", _p), ("n_tok", _i64),
                ("B", _i32), ("max_q_len", _i32), ("max_kv_len", _i32),
                ("max_pages_per_seq", _i32), ("n_logits", _i64), ("n_decode", _i32)]


_SIGS = {
    "bi_last_error": (ctypes.c_char_p, []),
    "bi_device_status": (_i32, [ctypes.POINTER(_i32), _i32, _p]),
    "bi_check_wait_bound": (_i32, [_i64, _p]),
    "bi_rmsnorm": (_i32, [_p, _p, _p, _i64, _i64, _f32, _p]),
    "bi_rmsnorm_f32in": (_i32, [_p, _p, _p, _i64, _i64, _f32, _p]),
    "bi_gemm": (_i32, [_p, _i64, _p, _i64, _p, _i64, _i32, _i64, _i64, _i64, _p]),
    "bi_gemm_f16": (_i32, [_p, _i64, _p, _i64, _p, _i64, _i32, _i64, _i64, _i64, _p]),
    "bi_gemm_swiglu": (_i32, [_p, _i64, _p, _i64, _p, _i64, _i64, _i64, _i64, _p]),
    "bi_gemm_qkv": (_i32, [_p, _i64, _p, _i64, _p, _i64, _i64, _i64, _i32, _i32, _p, _p, _i32, _p, _p, _p,
                           _i32, _p]),
    "bi_gemm_rmsnorm_workspace_size": (_i32, [_i64, _i64, ctypes.POINTER(_sz)]),
    "bi_gemm_rmsnorm": (_i32, [_p, _p, _f32, _p, _i64, _p, _i64, _i32, _i64, _i64, _i64, _p, _sz, _p]),
    "bi_gemm_rmsnorm_swiglu": (_i32, [_p, _p, _f32, _p, _i64, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "bi_kv_append": (_i32, [_p, _p, _i64, _p, _i64, _p, _p, ctypes.POINTER(KVLayout), _p]),
    "bi_attn_workspace_size": (_i32, [ctypes.POINTER(AttnShape), _i64, ctypes.POINTER(_sz)]),
    "bi_attn_decode": (_i32, [_p, _i64, _p, _p, _p, _p, _i32, ctypes.POINTER(AttnShape), _p,
                              _i64, _p, _sz, _p]),
    "bi_attn_decode_noalloc": (_i32, [_p, _i64, _p, _p, _p, _p, _i32, ctypes.POINTER(AttnShape),
                                      _p, _i64, _p]),
    "bi_attn_prefill": (_i32, [_p, _i64, _p, _i32, _i64, _p, _p, _p, _p, _i32,
                               ctypes.POINTER(AttnShape), _p, _i64, _p, _sz, _p]),
    "bi_gemm_x2": (_i32, [_p, _p, _i64, _p, _i64, _p, _i64, _i32, _i64, _i64, _i64, _p]),
    "bi_rmsnorm_split": (_i32, [_p, _p, _p, _p, _i64, _i64, _f32, _p]),
    "bi_split_bf16x2": (_i32, [_p, _i64, _p, _p, _p]),
    "bi_attn_f32_workspace_size": (_i32, [ctypes.POINTER(AttnShape), _i64, ctypes.POINTER(_sz)]),
    "bi_attn_f32": (_i32, [_p, _i64, _p, _i64, _p, _p, _p, _p, _i32, ctypes.POINTER(AttnShape), _p,
                           _i64, _p, _sz, _p]),
    "bi_embed": (_i32, [_p, _i64, _p, _i64, _i64, _p, _p]),
    "bi_rope_table": (_i32, [_p, _i32, _f64, _p]),
    "bi_rope": (_i32, [_p, _i64, _i32, _p, _i64, _p, _i32, _p]),
    "bi_swiglu": (_i32, [_p, _i64, _i64, _p, _p]),
    "bi_residual_add": (_i32, [_p, _p, _i64, _i64, _p]),
    "bi_argmax": (_i32, [_p, _i64, _i64, _i64, _p, _p]),
    "bi_model_create": (_i32, [ctypes.POINTER(ModelConfig), ctypes.POINTER(ModelWeights),
                               ctypes.POINTER(_p)]),
    "bi_model_destroy": (None, [_p]),
    "bi_forward_workspace_size": (_i32, [_p, _i64, _i64, _i32, ctypes.POINTER(_sz)]),
    "bi_forward": (_i32, [_p, ctypes.POINTER(Batch), _p, _p, _i32, _p, _p, _p, _sz, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTS = tuple(_SIGS)


class BIError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib.bi_last_error().decode(errors="replace")
        super().__init__(f"{fn} failed with status {status}: {msg}")


def _chk(fn: str, st: int) -> None:
    if st != BI_OK:
        raise BIError(fn, st)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int | None:
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    return torch.cuda.current_stream().cuda_stream


# ------------------------------------------------------------------ entry points

def bi_device_status(clear: bool = True, stream=None) -> int:
    v = _i32(0)
    st = lib.bi_device_status(ctypes.byref(v), int(clear), _stream(stream))
    if st not in (BI_OK, BI_ERR_DEVICE_CHECK):
        raise BIError("bi_device_status", st)
    return v.value


def bi_check_wait_bound(limit_cycles: int, stream=None) -> None:
    """Launches the wait-bound self-check (see include/bi.h)."""
    _chk("bi_check_wait_bound", lib.bi_check_wait_bound(int(limit_cycles), _stream(stream)))


def bi_rmsnorm(x, gamma, y, eps: float, stream=None) -> None:
    M, D = x.shape
    fn = "bi_rmsnorm_f32in" if x.dtype == torch.float32 else "bi_rmsnorm"
    _chk(fn, getattr(lib, fn)(_ptr(x), _ptr(gamma), _ptr(y), M, D, eps, _stream(stream)))


def bi_gemm(A, W, C, stream=None, add: bool = False) -> None:
    """C = A W^T (or, add=True with fp32 C, C += A W^T). A [M, K] bf16, W [N, K]
    bf16, C [M, N] bf16 or fp32 (row strides taken from the tensors). fp16 A
    and W go to bi_gemm_f16 (C fp16 or fp32)."""
    M, K = A.shape
    N = W.shape[0]
    f16 = A.dtype == torch.float16
    if (W.dtype == torch.float16) != f16:
        raise ValueError("bi_gemm: A and W must both be bf16 or both fp16")
    cdt = BI_F32 if C.dtype == torch.float32 else BI_BF16
    if cdt == BI_BF16 and C.dtype != A.dtype:
        raise ValueError("bi_gemm: a 16-bit C must have A's type")
    if add:
        if cdt != BI_F32:
            raise ValueError("bi_gemm(add=True) needs an fp32 C")
        cdt = BI_F32_ADD
    fn = "bi_gemm_f16" if f16 else "bi_gemm"
    _chk(fn, getattr(lib, fn)(_ptr(A), A.stride(0), _ptr(W), W.stride(0), _ptr(C), C.stride(0),
                              cdt, M, N, K, _stream(stream)))


def bi_gemm_rmsnorm_workspace_size(M: int, K: int) -> int:
    n = _sz(0)
    _chk("bi_gemm_rmsnorm_workspace_size", lib.bi_gemm_rmsnorm_workspace_size(M, K, ctypes.byref(n)))
    return n.value


def _check_fold_args(x, gamma, W, out, ws, rows_w: int, where: str) -> None:
    M, K = x.shape
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError(f"{where}: x must be contiguous fp32 [M, K]")
    if gamma.numel() < K or W.shape[0] < rows_w or W.shape[1] < K or out.shape[0] < M:
        raise ValueError(f"{where}: gamma / W / out smaller than the shapes")
    if ws.numel() * ws.element_size() < bi_gemm_rmsnorm_workspace_size(M, K):
        raise ValueError(f"{where}: workspace too small")


def bi_gemm_rmsnorm(x, gamma, eps: float, W, C, ws, c_dtype: int = BI_BF16, stream=None) -> None:
    """C = bi_gemm(bi_rmsnorm_f32in(x, gamma, eps), W) with the same bits. x [M, K]
    fp32, gamma [K] bf16, W [N, K] bf16, C [M, N] bf16 or fp32, ws from
    bi_gemm_rmsnorm_workspace_size(M, K)."""
    M, K = x.shape
    N = C.shape[1]
    _check_fold_args(x, gamma, W, C, ws, N, "bi_gemm_rmsnorm")
    _chk("bi_gemm_rmsnorm", lib.bi_gemm_rmsnorm(_ptr(x), _ptr(gamma), eps, _ptr(W), W.stride(0), _ptr(C),
                                                C.stride(0), c_dtype, M, N, K, _ptr(ws),
                                                ws.numel() * ws.element_size(), _stream(stream)))


def bi_gemm_rmsnorm_swiglu(x, gamma, eps: float, W, out, ws, stream=None) -> None:
    """out = bi_gemm_swiglu(bi_rmsnorm_f32in(x, gamma, eps), W) with the same
    bits. W [2F, K] bf16 (gate rows, then up rows), out [M, F] bf16."""
    M, K = x.shape
    F = out.shape[1]
    _check_fold_args(x, gamma, W, out, ws, 2 * F, "bi_gemm_rmsnorm_swiglu")
    _chk("bi_gemm_rmsnorm_swiglu", lib.bi_gemm_rmsnorm_swiglu(_ptr(x), _ptr(gamma), eps, _ptr(W), W.stride(0),
                                                              _ptr(out), out.stride(0), M, F, K, _ptr(ws),
                                                              ws.numel() * ws.element_size(), _stream(stream)))


def bi_gemm_swiglu(A, W, out, stream=None) -> None:
    """out = swiglu(A Wg^T, A Wu^T). A [M, K] bf16, W [2F, K] bf16 (gate rows,
    then up rows), out [M, F] bf16."""
    M, K = A.shape
    F = out.shape[1]
    if W.shape[0] != 2 * F:
        raise ValueError("bi_gemm_swiglu: W must have 2F rows")
    _chk("bi_gemm_swiglu", lib.bi_gemm_swiglu(_ptr(A), A.stride(0), _ptr(W), W.stride(0), _ptr(out),
                                              out.stride(0), M, F, K, _stream(stream)))


def bi_gemm_qkv(A, W, qkv, n_q_heads: int, n_kv_heads: int, positions, cos_sin, max_pos: int,
                slot_mapping, k_cache, v_cache, stream=None) -> None:
    """qkv = A W^T with RoPE on the q and k heads and k / v written to the
    paged caches (one layer's [num_pages, Hkv, ...] slices). A [M, K] bf16,
    W [(Hq + 2 Hkv) * 128, K] bf16, qkv [M, (Hq + 2 Hkv) * 128] bf16,
    positions / slot_mapping [M] int32, cos_sin the bi_rope_table of max_pos
    positions."""
    M, K = A.shape
    num_pages = k_cache.shape[0]
    _chk("bi_gemm_qkv", lib.bi_gemm_qkv(_ptr(A), A.stride(0), _ptr(W), W.stride(0), _ptr(qkv),
                                        qkv.stride(0), M, K, n_q_heads, n_kv_heads, _ptr(positions),
                                        _ptr(cos_sin), max_pos, _ptr(slot_mapping), _ptr(k_cache),
                                        _ptr(v_cache), num_pages, _stream(stream)))


def bi_gemm_x2(A_hi, A_lo, W, C, stream=None, add: bool = False) -> None:
    """C = (A_hi + A_lo) W^T (an fp32 activation carried as a bf16 pair)."""
    M, K = A_hi.shape
    N = W.shape[0]
    cdt = BI_F32 if C.dtype == torch.float32 else BI_BF16
    if add:
        if cdt != BI_F32:
            raise ValueError("bi_gemm_x2(add=True) needs an fp32 C")
        cdt = BI_F32_ADD
    _chk("bi_gemm_x2", lib.bi_gemm_x2(_ptr(A_hi), _ptr(A_lo), A_hi.stride(0), _ptr(W), W.stride(0),
                                      _ptr(C), C.stride(0), cdt, M, N, K, _stream(stream)))


def bi_rmsnorm_split(x, gamma, y_hi, y_lo, eps: float, stream=None) -> None:
    M, D = x.shape
    _chk("bi_rmsnorm_split", lib.bi_rmsnorm_split(_ptr(x), _ptr(gamma), _ptr(y_hi), _ptr(y_lo), M, D,
                                                  eps, _stream(stream)))


def bi_split_bf16x2(x, hi, lo, stream=None) -> None:
    _chk("bi_split_bf16x2", lib.bi_split_bf16x2(_ptr(x), x.numel(), _ptr(hi), _ptr(lo), _stream(stream)))


def bi_attn_f32(q, cu_q, k_cache, v_cache, block_table, seq_lens, shape: AttnShape, out, ws,
                stream=None) -> None:
    """fp32 attention; cu_q None means decode (one query per sequence)."""
    B = seq_lens.shape[0]
    _chk("bi_attn_f32", lib.bi_attn_f32(
        _ptr(q), q.stride(0), _ptr(cu_q), q.shape[0], _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
        _ptr(seq_lens), B, ctypes.byref(shape), _ptr(out), out.stride(0), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def bi_attn_f32_workspace_size(shape: AttnShape, max_tokens: int) -> int:
    n = _sz(0)
    _chk("bi_attn_f32_workspace_size", lib.bi_attn_f32_workspace_size(ctypes.byref(shape), max_tokens,
                                                                      ctypes.byref(n)))
    return n.value


def bi_kv_append(k_new, v_new, slot_mapping, k_cache, v_cache, stream=None) -> None:
    n_tok = k_new.shape[0]
    kv = KVLayout(k_cache.shape[0], k_cache.shape[1], HEAD_DIM, PAGE_SIZE)
    ld = k_new.stride(0)
    _chk("bi_kv_append", lib.bi_kv_append(_ptr(k_new), _ptr(v_new), ld, _ptr(slot_mapping), n_tok,
                                          _ptr(k_cache), _ptr(v_cache), ctypes.byref(kv),
                                          _stream(stream)))


def attn_shape(num_q_heads, num_kv_heads, num_pages, max_pages_per_seq, max_kv_len,
               scale=None) -> AttnShape:
    return AttnShape(num_q_heads, num_kv_heads, HEAD_DIM, PAGE_SIZE, num_pages,
                     max_pages_per_seq, max_kv_len,
                     1.0 / math.sqrt(HEAD_DIM) if scale is None else scale)


def bi_attn_workspace_size(shape: AttnShape, max_tokens: int) -> int:
    n = _sz(0)
    _chk("bi_attn_workspace_size", lib.bi_attn_workspace_size(ctypes.byref(shape), max_tokens,
                                                              ctypes.byref(n)))
    return n.value


def _check_attn_args(q, k_cache, v_cache, block_table, seq_lens, shape: AttnShape, out, n_rows: int,
                     where: str) -> None:
    """Host-side agreement of the tensors with the shape fields the kernels
    trust (the kernels range-check only what the device alone can see)."""
    B = seq_lens.shape[0]
    width = shape.num_q_heads * HEAD_DIM
    if q.shape[0] < n_rows or out.shape[0] < n_rows:
        raise ValueError(f"{where}: q / out have fewer than {n_rows} rows")
    if q.shape[-1] < width or out.shape[-1] < width or q.stride(-1) != 1 or out.stride(-1) != 1:
        raise ValueError(f"{where}: q / out rows must hold {width} contiguous elements")
    for name, c in (("k_cache", k_cache), ("v_cache", v_cache)):
        if c.shape[0] < shape.num_pages or not c.is_contiguous():
            raise ValueError(f"{where}: {name} holds fewer than num_pages={shape.num_pages} pages "
                             "or is not contiguous")
        if c.numel() < shape.num_pages * shape.num_kv_heads * PAGE_SIZE * HEAD_DIM:
            raise ValueError(f"{where}: {name} smaller than num_pages x num_kv_heads blocks")
    if block_table.dim() != 2 or block_table.shape[0] < B or block_table.shape[1] < shape.max_pages_per_seq \
            or block_table.stride(0) != shape.max_pages_per_seq or block_table.stride(1) != 1:
        raise ValueError(f"{where}: block_table must be [>= B, max_pages_per_seq] with row stride "
                         f"max_pages_per_seq={shape.max_pages_per_seq}")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError(f"{where}: block_table and seq_lens must be int32")


def bi_attn_decode(q, k_cache, v_cache, block_table, seq_lens, shape: AttnShape, out, ws,
                   stream=None) -> None:
    B = seq_lens.shape[0]
    _check_attn_args(q, k_cache, v_cache, block_table, seq_lens, shape, out, B, "bi_attn_decode")
    _chk("bi_attn_decode", lib.bi_attn_decode(
        _ptr(q), q.stride(0), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), B,
        ctypes.byref(shape), _ptr(out), out.stride(0), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def bi_attn_decode_noalloc(q, k_cache, v_cache, block_table, seq_lens, shape: AttnShape, out,
                           stream=None) -> None:
    """bi_attn_decode without a workspace argument: for callers that cannot
    allocate device memory; uses the library's fixed 16 MiB device scratch."""
    B = seq_lens.shape[0]
    _check_attn_args(q, k_cache, v_cache, block_table, seq_lens, shape, out, B, "bi_attn_decode_noalloc")
    _chk("bi_attn_decode_noalloc", lib.bi_attn_decode_noalloc(
        _ptr(q), q.stride(0), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), B,
        ctypes.byref(shape), _ptr(out), out.stride(0), _stream(stream)))


def bi_attn_prefill(q, cu_q, max_q_len: int, k_cache, v_cache, block_table, seq_lens,
                    shape: AttnShape, out, ws, stream=None) -> None:
    B = seq_lens.shape[0]
    _check_attn_args(q, k_cache, v_cache, block_table, seq_lens, shape, out, q.shape[0], "bi_attn_prefill")
    if cu_q.shape[0] < B + 1 or cu_q.dtype != torch.int32:
        raise ValueError("bi_attn_prefill: cu_q must be int32 with B + 1 entries")
    _chk("bi_attn_prefill", lib.bi_attn_prefill(
        _ptr(q), q.stride(0), _ptr(cu_q), max_q_len, q.shape[0], _ptr(k_cache), _ptr(v_cache),
        _ptr(block_table), _ptr(seq_lens), B, ctypes.byref(shape), _ptr(out), out.stride(0),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def bi_embed(tokens, table, out, stream=None) -> None:
    _chk("bi_embed", lib.bi_embed(_ptr(tokens), tokens.shape[0], _ptr(table), table.shape[0],
                                  table.shape[1], _ptr(out), _stream(stream)))


def bi_rope_table(cos_sin, max_pos: int, theta: float, stream=None) -> None:
    _chk("bi_rope_table", lib.bi_rope_table(_ptr(cos_sin), max_pos, theta, _stream(stream)))


def bi_rope(x, n_heads: int, positions, cos_sin, max_pos: int, stream=None) -> None:
    _chk("bi_rope", lib.bi_rope(_ptr(x), x.stride(0), n_heads, _ptr(positions), x.shape[0],
                                _ptr(cos_sin), max_pos, _stream(stream)))


def bi_swiglu(gu, out, stream=None) -> None:
    _chk("bi_swiglu", lib.bi_swiglu(_ptr(gu), gu.shape[0], gu.shape[1] // 2, _ptr(out),
                                    _stream(stream)))


def bi_residual_add(x, d, stream=None) -> None:
    _chk("bi_residual_add", lib.bi_residual_add(_ptr(x), _ptr(d), x.shape[0], x.shape[1],
                                                _stream(stream)))


def bi_argmax(logits, idx, stream=None) -> None:
    _chk("bi_argmax", lib.bi_argmax(_ptr(logits), logits.shape[0], logits.shape[1],
                                    logits.stride(0), _ptr(idx), _stream(stream)))


# ------------------------------------------------------------------ allocating helpers

def rmsnorm(x, gamma, eps: float):
    y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    bi_rmsnorm(x, gamma, y, eps)
    return y


def gemm(A, W, out_dtype=None):
    if out_dtype is None:
        out_dtype = A.dtype
    C = torch.empty((A.shape[0], W.shape[0]), dtype=out_dtype, device=A.device)
    bi_gemm(A, W, C)
    return C


def new_kv_cache(num_pages: int, num_kv_heads: int, device, n_layers: int = 1, zero=True,
                 precision: int = BI_PREC_BF16):
    """bf16 mode: k [L, pages, Hkv, 16, 128] and v [L, pages, Hkv, 128, 16] bf16
    (v transposed per page); the fp16 mode the same in fp16. fp32 modes: k and
    v [L, pages, Hkv, 16, 128] fp32."""
    f = torch.zeros if zero else torch.empty
    if precision in (BI_PREC_F32, BI_PREC_BF16_MLP):
        shp = (n_layers, num_pages, num_kv_heads, PAGE_SIZE, HEAD_DIM)
        return f(shp, dtype=torch.float32, device=device), f(shp, dtype=torch.float32, device=device)
    dt = torch.float16 if precision == BI_PREC_F16 else torch.bfloat16
    k = f((n_layers, num_pages, num_kv_heads, PAGE_SIZE, HEAD_DIM), dtype=dt, device=device)
    v = f((n_layers, num_pages, num_kv_heads, HEAD_DIM, PAGE_SIZE), dtype=dt, device=device)
    return k, v


class Model:
    """A bi_model handle over caller-owned device weights (dict of bf16 tensors
    in nn.Linear layout, as produced by synth.model_weights moved to the GPU)."""

    def __init__(self, cfg: dict, weights: dict):
        self.cfg = dict(cfg)
        self.weights = weights  # keep the tensors alive
        prec = cfg.get("precision", "bf16")
        self.precision = PRECISIONS[prec] if isinstance(prec, str) else int(prec)
        want = torch.float16 if self.precision == BI_PREC_F16 else torch.bfloat16
        bad = [n for n, _ in ModelWeights._fields_ if weights[n].dtype != want]
        if bad:
            raise ValueError(f"Model: weights {bad} must be {want} for precision {prec!r}")
        c = ModelConfig(cfg["n_layers"], cfg["d_model"], cfg["n_q_heads"], cfg["n_kv_heads"],
                        cfg["d_ff"], cfg["vocab"], cfg["max_pos"], cfg["rms_eps"],
                        cfg["rope_theta"], self.precision)
        w = ModelWeights(*[_ptr(weights[n]) for n, _ in ModelWeights._fields_])
        h = _p(0)
        _chk("bi_model_create", lib.bi_model_create(ctypes.byref(c), ctypes.byref(w),
                                                    ctypes.byref(h)))
        self.handle = h

    def __del__(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            lib.bi_model_destroy(self.handle)
            self.handle = None

    def workspace_size(self, max_tokens: int, max_logits: int, max_kv_len: int) -> int:
        n = _sz(0)
        _chk("bi_forward_workspace_size", lib.bi_forward_workspace_size(
            self.handle, max_tokens, max_logits, max_kv_len, ctypes.byref(n)))
        return n.value

    def forward(self, batch: dict, k_cache, v_cache, logits, next_tokens, ws, stream=None):
        """batch: device int32 tensors tokens, positions, slot_mapping, cu_q,
        seq_lens, block_table [B, P], logits_rows, plus host ints max_q_len,
        max_kv_len and (optional) n_decode: the number of leading one-token
        sequences."""
        bt = batch["block_table"]
        b = Batch(_ptr(batch["tokens"]), _ptr(batch["positions"]), _ptr(batch["slot_mapping"]),
                  _ptr(batch["cu_q"]), _ptr(batch["seq_lens"]), _ptr(bt),
                  _ptr(batch["logits_rows"]), batch["tokens"].shape[0],
                  batch["seq_lens"].shape[0], batch["max_q_len"], batch["max_kv_len"],
                  bt.shape[1], batch["logits_rows"].shape[0], batch.get("n_decode", 0))
        _chk("bi_forward", lib.bi_forward(self.handle, ctypes.byref(b), _ptr(k_cache),
                                          _ptr(v_cache), k_cache.shape[1], _ptr(logits),
                                          _ptr(next_tokens), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(stream)))
