"""Test helpers: read the sections of a prepared blob back into numpy arrays
in the oracle's canonical formats (pure data re-layout, no arithmetic of the
operator)."""
import numpy as np
import torch

from sparse_linear_layers_bitlinear_b200 import sbl


def _np(t):
    return t.detach().cpu().numpy()


def section(layer, name, nbytes):
    return _np(layer.section(name, nbytes))


def header_scalars(layer):
    L = layer.layout()
    raw = _np(layer.blob[L.header:L.header + 4096])
    gamma = raw[L.gamma - L.header:L.gamma - L.header + 4].view(np.float32)[0]
    g = raw[L.g - L.header:L.g - L.header + 4].view(np.float32)[0]
    status = raw[L.status - L.header:L.status - L.header + 4].view(np.uint32)[0]
    return gamma, g, status


def mask(layer):
    n_out, k, m = layer.n_out, layer.k, layer.m
    return section(layer, "mask", n_out * (k // m)).reshape(n_out, k // m)


def weff_from_bf16(layer):
    n_out, k = layer.n_out, layer.k
    raw = section(layer, "weff_bf16", n_out * k * 2).view(np.uint16).reshape(n_out, k)
    out = np.zeros((n_out, k), dtype=np.int8)
    out[raw == 0x3F80] = 1
    out[raw == 0xBF80] = -1
    bad = ~np.isin(raw, [0, 0x3F80, 0xBF80])
    assert not bad.any(), "weff_bf16 holds values outside {-1, 0, 1}"
    return out


def codes(layer):
    n_out, k = layer.n_out, layer.k
    return section(layer, "codes", n_out * k).view(np.int8).reshape(n_out, k)


def sp_values(layer):
    n_out, k = layer.n_out, layer.k
    return section(layer, "sp_values", n_out * k // 2).view(np.int8).reshape(n_out, k // 2)


def sp_meta_canonical(layer):
    """Tensor-core metadata re-laid out as [n_out, k/8] canonical nibble bytes,
    plus the padding region's bytes (rows >= n_out or k >= layer.k)."""
    n_out, k = layer.n_out, layer.k
    L = layer.layout()
    raw = section(layer, "sp_meta", int(L.sp_meta_bytes))
    kpad = (k + 255) // 256 * 256
    rpad = (n_out + 255) // 256 * 256
    kblocks = kpad // 128
    # [row_block][k_block][128 rows][16 bytes] -> [rpad][kpad/8]
    blocks = raw.reshape(rpad // 128, kblocks, 128, 16)
    full = blocks.transpose(0, 2, 1, 3).reshape(rpad, kblocks * 16)
    canonical = full[:n_out, : k // 8]
    pad_rows = full[n_out:, :]
    pad_cols = full[:n_out, k // 8:]
    return canonical, pad_rows, pad_cols


def gemv_bytes(layer):
    n_out, k = layer.n_out, layer.k
    return section(layer, "gemv", n_out * k // 4).reshape(n_out, k // 4)


def decode_gemv(gb):
    """(meta nibble [n_out, k/4], code0, code1) from the 2-bit decode packing."""
    nib = (gb >> 4) & 0xF
    to_code = np.array([0, 1, 0, -1], dtype=np.int8)  # 10 is never written
    c0 = to_code[gb & 3]
    c1 = to_code[(gb >> 2) & 3]
    return nib, c0, c1


def bf16_to_f64(t: torch.Tensor):
    return t.detach().float().cpu().numpy().astype(np.float64)
