"""Helpers shared by the GPU tests: move seeded bf16 inputs to the device, run the
CUDA path through the C ABI, and read results back."""
from __future__ import annotations

import numpy as np
import torch

import synthetic as sy


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> a bf16 CUDA tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> fp32 numpy (exact)."""
    bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return sy.bf16_bits_to_f32(bits)


def small_workload(M, C, Hq, Hkv, stride, causal, base="llama8b_gqa_32k", **kw):
    w = sy.workload(base)
    n_heavy = min(w.n_heavy or 16, M // 2)
    return w.with_(M=M, C=C, Hq=Hq, Hkv=Hkv, stride=stride, causal=causal, n_heavy=n_heavy, **kw)


def device_inputs(w, seed=sy.DEFAULT_SEED):
    Qb, Kb, Vb = sy.layer_inputs(w, seed)
    return (Qb, Kb, Vb), (to_dev(Qb), to_dev(Kb), to_dev(Vb))


def csr_to_dict(row_ptr: np.ndarray, col_idx: np.ndarray, bh: int, nb: int):
    """{r: kept array} for (batch*Hq + head) index bh."""
    return {r: col_idx[row_ptr[bh * nb + r]:row_ptr[bh * nb + r + 1]].astype(np.int64)
            for r in range(nb)}


def dict_to_csr(kept_by_bh, B, Hq, nb):
    """Oracle kept lists {(b, h): {r: kept}} -> device CSR in the library's row order."""
    lists = []
    for b in range(B):
        for h in range(Hq):
            k = kept_by_bh[(b, h)]
            lists += [np.asarray(k[r], np.int32) for r in range(nb)]
    counts = np.array([len(x) for x in lists], np.int64)
    row_ptr = np.zeros(len(lists) + 1, np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col = np.concatenate(lists).astype(np.int32)
    return (torch.from_numpy(row_ptr.astype(np.int32)).cuda(), torch.from_numpy(col).cuda())


def poison_(t: torch.Tensor) -> torch.Tensor:
    """Fill an output buffer with values no kernel writes (NaN for floating point,
    -7 for int32, 0xFF bytes for raw workspaces), so that an element a kernel never
    writes cannot pass for a result left behind by an earlier call."""
    if t.dtype.is_floating_point:
        t.fill_(float("nan"))
    elif t.dtype == torch.uint8:
        t.fill_(0xFF)
    else:
        t.fill_(-7)
    return t


def poisoned(shape, dtype=torch.float32, device="cuda") -> torch.Tensor:
    return poison_(torch.empty(shape, dtype=dtype, device=device))


def poisoned_like(t: torch.Tensor) -> torch.Tensor:
    return poison_(torch.empty_like(t))


def poison_buffers(bufs):
    """poison_ every tensor of a Buffers set (outputs and workspaces)."""
    for name in ("scores", "score_ws", "select_ws", "row_ptr", "col_idx", "nnz", "O", "lse"):
        t = getattr(bufs, name)
        if t is not None:
            poison_(t)
    return bufs
