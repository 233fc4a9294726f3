"""Sparse-BitLinear CPU oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct CPU implementation of the Sparse-BitLinear
operator (arXiv 2603.05168, "Sparse-BitNet: 1.58-bit LLMs are Naturally
Friendly to Semi-Structured Sparsity").  Only the test suite, the smoke check
and the benchmark's CPU-baseline leg may import it.  It shares no code with
the CUDA library and never imports it.

The arithmetic lives in ``sbl_oracle.cpp`` (plain C++ loops); this module
only marshals numpy arrays into it.  Every function names the step of the
operator it computes:

  A1 absmean scale            absmean_gamma / clamped_scale
  A2 N:M magnitude mask       nm_mask
  A3 ternarise, mask, pack    ternary, apply_mask, pack24, pack_nm, pack24_code6
  A4 per-token int8 absmax    act_quant
  A5 int32 product            gemm_acc, acc_at
  A6 dequant rescale          dequant
  A7 STE input gradient       grad_x, grad_x_at
  A8 dense weight gradient    grad_w, grad_w_at

Parity status: every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` against closed forms, exact rational arithmetic,
library routines or brute force; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sbl_oracle.cpp")
_LIB = os.path.join(_HERE, "libsbl_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with plain IEEE semantics (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "sbl_oracle.h"))
    ):
        cmd = [
            "g++", "-std=c++17", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
            "-shared", "-fPIC", "-o", _LIB, _SRC,
        ]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I = ctypes.c_int
    F = ctypes.c_float
    sig = {
        "sbo_absmean_bits": (ctypes.c_uint32, [P, I64]),
        "sbo_clamped_scale": (F, [F]),
        "sbo_nm_mask": (None, [P, I64, I64, I, I, P]),
        "sbo_nm_mask_from_codes": (None, [P, I64, I64, I, I, P]),
        "sbo_ternary": (None, [P, I64, F, P]),
        "sbo_apply_mask": (None, [P, P, I64, I64, I, P]),
        "sbo_pack24": (None, [P, P, I64, I64, P, P]),
        "sbo_pack_nm": (None, [P, P, I64, I64, I, I, P, P]),
        "sbo_pack24_code6": (None, [P, P, I64, I64, P]),
        "sbo_act_quant": (None, [P, I64, I64, P, P]),
        "sbo_gemm_acc": (I, [P, P, I64, I64, I64, P]),
        "sbo_acc_at": (ctypes.c_int32, [P, P, I64]),
        "sbo_dequant": (None, [P, P, F, I64, I64, P]),
        "sbo_grad_x": (None, [P, P, F, I64, I64, I64, P]),
        "sbo_grad_x_at": (ctypes.c_double, [P, P, F, I64, I64, I64, I64]),
        "sbo_grad_w": (None, [P, P, I64, I64, I64, P]),
        "sbo_grad_w_at": (ctypes.c_double, [P, P, I64, I64, I64, I64, I64]),
        "sbo_grad_w_masked": (None, [P, P, P, I64, I64, I64, I, P]),
        "sbo_round_bf16": (None, [P, I64, P]),
        "sbo_dequant_act": (None, [P, P, I64, I64, P]),
        "sbo_threads": (I, []),
        "sbo_set_threads": (None, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    """bf16 data as its uint16 bit patterns (accepts a torch bf16 tensor or uint16 array)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch  # local: torch is only needed when a tensor is passed

        return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def threads() -> int:
    return int(_load().sbo_threads())


def set_threads(n: int) -> None:
    """Set the OpenMP thread count for later oracle calls; results do not depend on it."""
    _load().sbo_set_threads(int(n))


def absmean_gamma(w) -> np.float32:
    """A1: gamma = RN_fp32(sum|w| / numel), exact sum over all master weights."""
    w = _u16(w)
    bits = _load().sbo_absmean_bits(_ptr(w), w.size)
    return np.array([bits], dtype=np.uint32).view(np.float32)[0]


def clamped_scale(gamma) -> np.float32:
    """g = max(gamma, 1e-5)."""
    return np.float32(_load().sbo_clamped_scale(float(gamma)))


def nm_mask(w, n: int, m: int) -> np.ndarray:
    """A2: uint8 [n_out, k/m]; bit j set when position j of the group is kept."""
    w = _u16(w)
    n_out, k = w.shape
    out = np.zeros((n_out, k // m), dtype=np.uint8)
    _load().sbo_nm_mask(_ptr(w), n_out, k, n, m, _ptr(out))
    return out


def nm_mask_from_codes(q: np.ndarray, n: int, m: int) -> np.ndarray:
    """Ablation of A2 ([de] §4, [fr] §5): the mask from |q| instead of |w|."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    n_out, k = q.shape
    out = np.zeros((n_out, k // m), dtype=np.uint8)
    _load().sbo_nm_mask_from_codes(_ptr(q), n_out, k, n, m, _ptr(out))
    return out


def ternary(w, g) -> np.ndarray:
    """A3: int8 codes in {-1, 0, 1}, before the mask."""
    w = _u16(w)
    out = np.zeros(w.shape, dtype=np.int8)
    _load().sbo_ternary(_ptr(w), w.size, float(g), _ptr(out))
    return out


def apply_mask(q: np.ndarray, mask: np.ndarray, m: int) -> np.ndarray:
    """A3: weff = q * mask (quant first, then mask)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    n_out, k = q.shape
    out = np.zeros_like(q)
    _load().sbo_apply_mask(_ptr(q), _ptr(mask), n_out, k, m, _ptr(out))
    return out


def pack24(weff: np.ndarray, mask: np.ndarray):
    """Canonical 2:4 packing: (vals int8 [n_out, k/2], meta uint8 [n_out, k/8])."""
    weff = np.ascontiguousarray(weff, dtype=np.int8)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    n_out, k = weff.shape
    vals = np.zeros((n_out, k // 2), dtype=np.int8)
    meta = np.zeros((n_out, k // 8), dtype=np.uint8)
    _load().sbo_pack24(_ptr(weff), _ptr(mask), n_out, k, _ptr(vals), _ptr(meta))
    return vals, meta


def pack_nm(weff: np.ndarray, mask: np.ndarray, n: int, m: int):
    """Compressed-index decode pack of any N:M (blocks of 8 weights): returns
    (masks8 [n_out, k/8] uint8, codes [n_out, k*n/(4m)] uint8), the kept
    2-bit codes of each row in index order, least significant bit first."""
    weff = np.ascontiguousarray(weff, dtype=np.int8)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    n_out, k = weff.shape
    assert k % 64 == 0
    masks8 = np.empty((n_out, k // 8), dtype=np.uint8)
    codes = np.empty((n_out, k * n // (4 * m)), dtype=np.uint8)
    _load().sbo_pack_nm(_ptr(weff), _ptr(mask), n_out, k, n, m, _ptr(masks8), _ptr(codes))
    return masks8, codes


def pack24_code6(weff: np.ndarray, mask: np.ndarray):
    """The 6-bit 2:4 group code (54 states, 1.5 bits a weight): uint8
    [n_out, 3k/16], one least-significant-bit-first stream of 6-bit states per
    row, state = 9 p + 3 d(c_i0) + d(c_i1) (p: rank of the kept pair, d: code
    mod 3)."""
    weff = np.ascontiguousarray(weff, dtype=np.int8)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    n_out, k = weff.shape
    assert k % 16 == 0
    out = np.empty((n_out, k * 6 // 32), dtype=np.uint8)
    _load().sbo_pack24_code6(_ptr(weff), _ptr(mask), n_out, k, _ptr(out))
    return out


def act_quant(x):
    """A4: (xq int8 [t, k], a' fp32 [t])."""
    x = _u16(x)
    t, k = x.shape
    xq = np.zeros((t, k), dtype=np.int8)
    ap = np.zeros((t,), dtype=np.float32)
    _load().sbo_act_quant(_ptr(x), t, k, _ptr(xq), _ptr(ap))
    return xq, ap


def gemm_acc(xq: np.ndarray, weff: np.ndarray) -> np.ndarray:
    """A5: int32 [t, n_out] = xq . weff^T, accumulated in int64."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    weff = np.ascontiguousarray(weff, dtype=np.int8)
    t, k = xq.shape
    n_out = weff.shape[0]
    out = np.zeros((t, n_out), dtype=np.int32)
    rc = _load().sbo_gemm_acc(_ptr(xq), _ptr(weff), t, n_out, k, _ptr(out))
    if rc != 0:
        raise OverflowError("accumulator outside int32")
    return out


def acc_at(xq: np.ndarray, weff: np.ndarray, ti: int, o: int) -> int:
    xr = np.ascontiguousarray(xq[ti], dtype=np.int8)
    wr = np.ascontiguousarray(weff[o], dtype=np.int8)
    return int(_load().sbo_acc_at(_ptr(xr), _ptr(wr), xr.size))


def dequant(acc: np.ndarray, a_prime: np.ndarray, g) -> np.ndarray:
    """A6: fp32 y = (float)acc * ((g * a') / 127)."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    a_prime = np.ascontiguousarray(a_prime, dtype=np.float32)
    t, n_out = acc.shape
    y = np.zeros((t, n_out), dtype=np.float32)
    _load().sbo_dequant(_ptr(acc), _ptr(a_prime), float(g), t, n_out, _ptr(y))
    return y


def grad_x(dy, weff: np.ndarray, g) -> np.ndarray:
    """A7: fp64 dX = g * (dY . weff)."""
    dy = _u16(dy)
    weff = np.ascontiguousarray(weff, dtype=np.int8)
    t, n_out = dy.shape
    k = weff.shape[1]
    out = np.zeros((t, k), dtype=np.float64)
    _load().sbo_grad_x(_ptr(dy), _ptr(weff), float(g), t, n_out, k, _ptr(out))
    return out


def grad_x_at(dy, weff: np.ndarray, g, ti: int, ki: int) -> float:
    dy = _u16(dy)
    weff = np.ascontiguousarray(weff, dtype=np.int8)
    t, n_out = dy.shape
    return float(_load().sbo_grad_x_at(_ptr(dy), _ptr(weff), float(g), n_out, weff.shape[1], ti, ki))


def grad_w(dy, x) -> np.ndarray:
    """A8: fp64 dW = dY^T . X over every master weight."""
    dy = _u16(dy)
    x = _u16(x)
    t, n_out = dy.shape
    k = x.shape[1]
    out = np.zeros((n_out, k), dtype=np.float64)
    _load().sbo_grad_w(_ptr(dy), _ptr(x), t, n_out, k, _ptr(out))
    return out


def grad_w_at(dy, x, oi: int, ki: int) -> float:
    dy = _u16(dy)
    x = _u16(x)
    t, n_out = dy.shape
    return float(_load().sbo_grad_w_at(_ptr(dy), _ptr(x), t, n_out, x.shape[1], oi, ki))


def grad_w_masked(dy, x, mask: np.ndarray, m: int) -> np.ndarray:
    """Ablation of A8 ([de] §4, [fr] §5): dW with the gradient of pruned weights blocked."""
    dy, x = _u16(dy), _u16(x)
    t, n_out = dy.shape
    k = x.shape[1]
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    out = np.zeros((n_out, k), dtype=np.float64)
    _load().sbo_grad_w_masked(_ptr(dy), _ptr(x), _ptr(mask), t, n_out, k, m, _ptr(out))
    return out


def dequant_act(xq: np.ndarray, a_prime: np.ndarray) -> np.ndarray:
    """dW operand of the detach-form STE: xhat = RN_bf16(xq * a' / 127), bf16 bits [t, k]."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    ap = np.ascontiguousarray(a_prime, dtype=np.float32)
    t, k = xq.shape
    out = np.zeros((t, k), dtype=np.uint16)
    _load().sbo_dequant_act(_ptr(xq), _ptr(ap), t, k, _ptr(out))
    return out


def grad_w_quant_x(dy, x) -> np.ndarray:
    """dW = dY^T . xhat, xhat the dequantised activations of x (SBL_DW_QUANT_X reading)."""
    xq, ap = act_quant(x)
    return grad_w(dy, dequant_act(xq, ap))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.zeros(a.shape, dtype=np.uint16)
    _load().sbo_round_bf16(_ptr(a), a.size, _ptr(out))
    return out


def prepare(w, n: int, m: int, mask_from_codes: bool = False):
    """A1-A3 in the pages' order: returns dict(gamma, g, mask, q, weff).
    mask_from_codes: the pages' ablation that builds the mask from |q|."""
    w = _u16(w)
    gamma = absmean_gamma(w)
    g = clamped_scale(gamma)
    q = ternary(w, g)
    mask = nm_mask_from_codes(q, n, m) if mask_from_codes else nm_mask(w, n, m)
    weff = apply_mask(q, mask, m)
    return {"gamma": gamma, "g": g, "mask": mask, "q": q, "weff": weff}


def forward(w, x, n: int, m: int, mask_from_codes: bool = False):
    """A1-A6: returns dict with the prepare outputs plus xq, a_prime, acc, y."""
    p = prepare(w, n, m, mask_from_codes)
    xq, ap = act_quant(x)
    acc = gemm_acc(xq, p["weff"])
    y = dequant(acc, ap, p["g"])
    p.update({"xq": xq, "a_prime": ap, "acc": acc, "y": y})
    return p
