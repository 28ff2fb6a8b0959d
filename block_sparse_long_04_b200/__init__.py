"""XAttention block-sparse prefill attention for NVIDIA B200 (sm_100a).

A thin ctypes binding over libxattn.so (C ABI in include/xattn.h). Each function
has the name of the C entry point it calls and does argument marshalling only:
shapes are read from the torch tensors, pointers and the current CUDA stream are
passed through, and the status code is turned into an exception. Every step of
the computation runs in the library's CUDA kernels; there is no fallback. If the
library is missing or fails to load, the first call into it raises ImportError.

The method (page title, section):
- DuSA rebuttal (paperhub tM5mjMfFmS), Response to Q2: strided reshape of Q and K
  to (B, H, M//stride, stride*C) with a softmax over the last two dimensions.
- XAttention abstract (arXiv 2503.16428): antidiagonal sums (lower-left to
  upper-right) as the block-importance proxy.
- XAttention summary (atlas.scime.ai), Approach: keep the minimal set of blocks
  whose softmax-normalised antidiagonal mass reaches a per-head threshold.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libxattn.so")

XATTN_OK, XATTN_EINVAL, XATTN_ECAPACITY, XATTN_ECUDA, XATTN_ETIMEOUT, XATTN_EUNSUPPORTED = range(6)

# name -> (restype, argtypes); mirrors include/xattn.h
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "xattn_status_string": (ctypes.c_char_p, [_I]),
    "xattn_version": (_I, []),
    "xattn_score_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "xattn_score": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _Z, _P]),
    "xattn_select_workspace_size": (_Z, [_I, _I, _I]),
    "xattn_select": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _Z, _P, _P, _Z, _P]),
    "xattn_sparse_attn": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P]),
    "xattn_dense_attn": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P]),
    "xattn_get_device_error": (_I, [_P]),
    "xattn_select_noalloc": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _Z, _P, _P]),
    "xattn_score_ex": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _Z, _P]),
    "xattn_select_ex": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _Z, _P, _P, _Z, _P]),
    "xattn_selftest_wait_timeout": (_I, [ctypes.c_longlong, _P, _P]),
    "xattn_selftest_exp2": (_I, [_P, _P, ctypes.c_longlong, _P]),
    "xattn_select_group_workspace_size": (_Z, [_I, _I, _I, _I]),
    "xattn_select_group": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P, _P, _Z, _P]),
    "xattn_sparse_attn_group": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P,
                                     _P]),
    "xattn_score_select_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "xattn_score_select": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _I, _P, _P, _P, _Z,
                                _P, _P, _Z, _P]),
}

XATTN_PATTERN_ANTIDIAGONAL, XATTN_PATTERN_DIAGONAL = 0, 1
XATTN_SELECT_THRESHOLD, XATTN_SELECT_TOPK, XATTN_SELECT_RATIO = 0, 1, 2


class XAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libxattn.so not found at {LIB_PATH}; build it with "
            "`python -m block_sparse_long_04_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


class _Lazy:
    """Loads libxattn.so on first use; a missing library raises ImportError then."""
    _cdll = None

    def __getattr__(self, name):
        if _Lazy._cdll is None:
            _Lazy._cdll = _load()
        return getattr(_Lazy._cdll, name)


_lib = _Lazy()


def status_string(status: int) -> str:
    return _lib.xattn_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != XATTN_OK:
        raise XAttnError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _bf16(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16:
            raise TypeError("Q, K, V, O must be bfloat16")


# ------------------------------------------------------------------ sizes
def xattn_score_workspace_size(B: int, Hq: int, M: int, stride: int, causal: bool,
                               block: int = 128) -> int:
    """Bytes of the scoring workspace; sized for the `causal` flag of the call."""
    return int(_lib.xattn_score_workspace_size(B, Hq, M, stride, block, int(causal)))


def xattn_select_workspace_size(B: int, Hq: int, nb: int) -> int:
    return int(_lib.xattn_select_workspace_size(B, Hq, nb))


# ------------------------------------------------------------ entry points
def xattn_score(Q, K, stride: int, causal: bool, score_scale: float, scores, workspace,
                block: int = 128, stream=None) -> None:
    """scores[B,Hq,nb,nb] (fp32) <- strided antidiagonal block scores of Q, K."""
    _dev(Q, K, scores, workspace)
    _bf16(Q, K)
    B, Hq, M, C = Q.shape
    Hkv = K.shape[1]
    rc = _lib.xattn_score(_ptr(Q), _ptr(K), B, Hq, Hkv, M, C, stride, block, int(causal),
                          float(score_scale), _ptr(scores), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "xattn_score")


def xattn_score_ex(Q, K, stride: int, causal: bool, pattern: int, score_scale: float, scores,
                   workspace, block: int = 128, stream=None) -> None:
    """xattn_score with a pattern: XATTN_PATTERN_ANTIDIAGONAL or XATTN_PATTERN_DIAGONAL."""
    _dev(Q, K, scores, workspace)
    _bf16(Q, K)
    B, Hq, M, C = Q.shape
    Hkv = K.shape[1]
    rc = _lib.xattn_score_ex(_ptr(Q), _ptr(K), B, Hq, Hkv, M, C, stride, block, int(causal),
                             int(pattern), float(score_scale), _ptr(scores), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "xattn_score_ex")


def xattn_select_ex(scores, param, rule: int, causal: bool, row_ptr, col_idx, nnz, workspace,
                    stream=None) -> None:
    """Selection by XATTN_SELECT_THRESHOLD (param = tau), XATTN_SELECT_TOPK (param = k)
    or XATTN_SELECT_RATIO (param = fraction of the candidates)."""
    _dev(scores, param, row_ptr, col_idx, nnz, workspace)
    B, Hq, nb, _ = scores.shape
    rc = _lib.xattn_select_ex(_ptr(scores), _ptr(param), int(rule), B, Hq, nb, int(causal),
                              _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(nnz),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _check(rc, "xattn_select_ex")


def xattn_select_group_workspace_size(B: int, Hq: int, Hkv: int, nb: int) -> int:
    return int(_lib.xattn_select_group_workspace_size(B, Hq, Hkv, nb))


def xattn_select_group(scores, param, rule: int, Hkv: int, causal: bool, row_ptr, col_idx, nnz,
                       workspace, stream=None) -> None:
    """GQA-shared kept lists (a variant): per (b, kv head, query block) the union of
    the group's per-head selections; CSR over B*Hkv*nb rows."""
    _dev(scores, param, row_ptr, col_idx, nnz, workspace)
    B, Hq, nb, _ = scores.shape
    rc = _lib.xattn_select_group(_ptr(scores), _ptr(param), int(rule), B, Hq, Hkv, nb,
                                 int(causal), _ptr(row_ptr), _ptr(col_idx), col_idx.numel(),
                                 _ptr(nnz), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "xattn_select_group")


def xattn_score_select_workspace_size(B: int, Hq: int, M: int, stride: int, causal: bool,
                                      block: int = 128) -> int:
    return int(_lib.xattn_score_select_workspace_size(B, Hq, M, stride, block, int(causal)))


def xattn_score_select(Q, K, param, rule: int, stride: int, causal: bool, score_scale: float, scores,
                       row_ptr, col_idx, nnz, workspace, block: int = 128, stream=None) -> None:
    """Scores and kept lists in one fused pass (same results as xattn_score followed
    by xattn_select_ex)."""
    _dev(Q, K, param, scores, row_ptr, col_idx, nnz, workspace)
    _bf16(Q, K)
    B, Hq, M, C = Q.shape
    Hkv = K.shape[1]
    rc = _lib.xattn_score_select(_ptr(Q), _ptr(K), B, Hq, Hkv, M, C, stride, block, int(causal),
                                 float(score_scale), _ptr(param), int(rule), _ptr(scores),
                                 _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(nnz),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(rc, "xattn_score_select")


def xattn_select(scores, tau, causal: bool, row_ptr, col_idx, nnz, workspace, stream=None) -> None:
    """CSR (row_ptr, col_idx, nnz) <- per-head threshold selection of scores."""
    _dev(scores, tau, row_ptr, col_idx, nnz, workspace)
    B, Hq, nb, _ = scores.shape
    rc = _lib.xattn_select(_ptr(scores), _ptr(tau), B, Hq, nb, int(causal), _ptr(row_ptr),
                           _ptr(col_idx), col_idx.numel(), _ptr(nnz), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "xattn_select")


def xattn_select_noalloc(scores, tau, causal: bool, row_ptr, col_idx, nnz, stream=None) -> None:
    """xattn_select without a workspace, for callers that cannot allocate device
    memory while this step runs: the library keeps a fixed scratch array of
    XATTN_SELECT_NOALLOC_MAX_ROWS rows per device. Calls that overlap on the GPU
    race on that array, so issue them on one stream."""
    _dev(scores, tau, row_ptr, col_idx, nnz)
    B, Hq, nb, _ = scores.shape
    rc = _lib.xattn_select_noalloc(_ptr(scores), _ptr(tau), B, Hq, nb, int(causal), _ptr(row_ptr),
                                   _ptr(col_idx), col_idx.numel(), _ptr(nnz), _stream(stream))
    _check(rc, "xattn_select_noalloc")


XATTN_SELECT_NOALLOC_MAX_ROWS = 262144


def xattn_sparse_attn(Q, K, V, row_ptr, col_idx, causal: bool, softmax_scale: float, O,
                      lse=None, block: int = 128, stream=None) -> None:
    """O <- softmax attention of Q over the kept key blocks listed in the CSR."""
    _dev(Q, K, V, row_ptr, col_idx, O, lse)
    _bf16(Q, K, V, O)
    B, Hq, M, C = Q.shape
    Hkv = K.shape[1]
    rc = _lib.xattn_sparse_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(row_ptr), _ptr(col_idx), B, Hq,
                                Hkv, M, C, block, int(causal), float(softmax_scale), _ptr(O),
                                _ptr(lse), _stream(stream))
    _check(rc, "xattn_sparse_attn")


def xattn_sparse_attn_group(Q, K, V, row_ptr, col_idx, causal: bool, softmax_scale: float, O,
                            lse=None, block: int = 128, stream=None) -> None:
    """xattn_sparse_attn over GQA-shared lists (CSR rows per batch, KV head, query block)."""
    _dev(Q, K, V, row_ptr, col_idx, O, lse)
    _bf16(Q, K, V, O)
    B, Hq, M, C = Q.shape
    Hkv = K.shape[1]
    rc = _lib.xattn_sparse_attn_group(_ptr(Q), _ptr(K), _ptr(V), _ptr(row_ptr), _ptr(col_idx), B,
                                      Hq, Hkv, M, C, block, int(causal), float(softmax_scale),
                                      _ptr(O), _ptr(lse), _stream(stream))
    _check(rc, "xattn_sparse_attn_group")


def xattn_dense_attn(Q, K, V, causal: bool, softmax_scale: float, O, lse=None, block: int = 128,
                     stream=None) -> None:
    """O <- softmax attention of Q over every key block (dense baseline)."""
    _dev(Q, K, V, O, lse)
    _bf16(Q, K, V, O)
    B, Hq, M, C = Q.shape
    Hkv = K.shape[1]
    rc = _lib.xattn_dense_attn(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, M, C, block, int(causal),
                               float(softmax_scale), _ptr(O), _ptr(lse), _stream(stream))
    _check(rc, "xattn_dense_attn")


def xattn_selftest_wait_timeout(limit_ns: int, timed_out, stream=None) -> None:
    """Diagnostic: a device wait that nothing completes must give up after
    limit_ns and raise XATTN_ETIMEOUT (read it with xattn_get_device_error)."""
    _dev(timed_out)
    _check(_lib.xattn_selftest_wait_timeout(int(limit_ns), _ptr(timed_out), _stream(stream)),
           "xattn_selftest_wait_timeout")


def xattn_selftest_exp2(x, y, stream=None) -> None:
    """y = 2^x through the FMA-pipe exponential of the attention softmax."""
    _dev(x, y)
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise ValueError("x and y must be float32 tensors of the same size")
    _check(_lib.xattn_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)),
           "xattn_selftest_exp2")


def xattn_get_device_error(stream=None) -> int:
    return int(_lib.xattn_get_device_error(_stream(stream)))


# ------------------------------------------------------ pipeline helpers
def max_kept(B: int, Hq: int, nb: int, causal: bool) -> int:
    """Worst-case number of kept entries (every candidate of every row)."""
    return B * Hq * (nb * (nb + 1) // 2 if causal else nb * nb)


@dataclass
class Buffers:
    """Device buffers for one prefill layer (allocated once, reused)."""
    scores: torch.Tensor
    score_ws: torch.Tensor
    select_ws: torch.Tensor
    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    nnz: torch.Tensor
    O: torch.Tensor
    lse: Optional[torch.Tensor]

    @staticmethod
    def allocate(B, Hq, M, C, stride, causal, block=128, device="cuda", with_lse=False,
                 col_capacity=None):
        nb = M // block
        dev = torch.device(device)
        cap = max_kept(B, Hq, nb, causal) if col_capacity is None else col_capacity
        return Buffers(
            scores=torch.empty((B, Hq, nb, nb), dtype=torch.float32, device=dev),
            # sized for the fused score+select call, which also serves xattn_score
            score_ws=torch.empty(max(1, xattn_score_select_workspace_size(B, Hq, M, stride, causal,
                                                                          block)),
                                 dtype=torch.uint8, device=dev),
            select_ws=torch.empty(max(1, xattn_select_workspace_size(B, Hq, nb)),
                                  dtype=torch.uint8, device=dev),
            row_ptr=torch.empty(B * Hq * nb + 1, dtype=torch.int32, device=dev),
            col_idx=torch.empty(max(1, cap), dtype=torch.int32, device=dev),
            nnz=torch.zeros(1, dtype=torch.int32, device=dev),
            O=torch.empty((B, Hq, M, C), dtype=torch.bfloat16, device=dev),
            lse=torch.empty((B, Hq, M), dtype=torch.float32, device=dev) if with_lse else None,
        )


def default_score_scale(stride: int, C: int) -> float:
    """1/sqrt(stride*C): the usual attention scale for the reshaped width stride*C."""
    return 1.0 / math.sqrt(stride * C)


def xattn_prefill(Q, K, V, tau, stride: int, causal: bool, bufs: Buffers,
                  score_scale: Optional[float] = None, softmax_scale: Optional[float] = None,
                  block: int = 128, stream=None) -> torch.Tensor:
    """score -> select -> sparse attention on one stream; returns bufs.O.

    Scoring and selection run as two calls: on B200 that is faster than the fused
    xattn_score_select, whose in-kernel ranking runs on one CTA per SM behind the
    scoring tile."""
    C = Q.shape[-1]
    ss = default_score_scale(stride, C) if score_scale is None else score_scale
    sa = 1.0 / math.sqrt(C) if softmax_scale is None else softmax_scale
    xattn_score(Q, K, stride, causal, ss, bufs.scores, bufs.score_ws, block, stream)
    xattn_select(bufs.scores, tau, causal, bufs.row_ptr, bufs.col_idx, bufs.nnz, bufs.select_ws,
                 stream)
    xattn_sparse_attn(Q, K, V, bufs.row_ptr, bufs.col_idx, causal, sa, bufs.O, bufs.lse, block,
                      stream)
    return bufs.O
