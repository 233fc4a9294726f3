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
    """The interleaved 2:4 decode pack of a layer re-laid out as its canonical
    [n_out, k/4] group bytes (units of 16 rows x 128 k: lane (row % 8) * 4 + t
    holds 8 bytes of its row, then 8 of the row 8 below, for the groups
    8t..8t+7 of the unit), plus every byte outside the matrix."""
    n_out, k = layer.n_out, layer.k
    tiles, upr = (n_out + 15) // 16, (k + 127) // 128
    L = layer.layout()
    assert L.gemv_bytes == tiles * upr * 512
    raw = section(layer, "gemv", int(L.gemv_bytes)).reshape(tiles, upr, 8, 4, 2, 8)  # tile, unit, g, t, hi, byte
    full = raw.transpose(0, 4, 2, 1, 3, 5).reshape(tiles * 16, upr * 32)
    pad = np.concatenate([full[n_out:].ravel(), full[:n_out, k // 4:].ravel()])
    return full[:n_out, :k // 4], pad


def gemv_code6(layer):
    """The 6-bit 2:4 decode pack of a layer re-laid out as the oracle's
    per-row streams [n_out, 3k/16] (units of 16 rows x 128 k, 384 bytes: word
    j of slot 4 (row % 8) + t in plane j; a slot's 96 bits are the 48 of row r
    for groups 8t..8t+7, then the 48 of row r + 8), plus every byte outside the
    matrix."""
    n_out, k = layer.n_out, layer.k
    tiles, upr = (n_out + 15) // 16, (k + 127) // 128
    L = layer.layout()
    assert L.gemv_bytes == tiles * upr * 384
    raw = section(layer, "gemv", int(L.gemv_bytes)).reshape(tiles, upr, 3, 32, 4)  # tile, unit, plane, slot, byte
    slots = raw.transpose(0, 1, 3, 2, 4).reshape(tiles, upr, 8, 4, 2, 6)  # tile, unit, g, t, hi, byte
    full = slots.transpose(0, 4, 2, 1, 3, 5).reshape(tiles * 16, upr * 24)
    row_bytes = 3 * k // 16
    pad = np.concatenate([full[n_out:].ravel(), full[:n_out, row_bytes:].ravel()])
    return full[:n_out, :row_bytes], pad


def decode_gemv(gb):
    """(meta nibble [n_out, k/4], code0, code1) from the 2-bit decode packing."""
    nib = (gb >> 4) & 0xF
    to_code = np.array([0, 1, 0, -1], dtype=np.int8)  # 10 is never written
    c0 = to_code[gb & 3]
    c1 = to_code[(gb >> 2) & 3]
    return nib, c0, c1


def nm_pack_fields(masks8, codes, n, m):
    """The oracle's canonical compressed-index pack as (mask bytes [n_out, k/8],
    code fields [n_out, k/8]): field b is the 2 n8 bits of block b's kept codes."""
    n8 = 8 * n // m
    n_out, blocks = masks8.shape
    bits = np.unpackbits(codes, axis=1, bitorder="little").reshape(n_out, blocks, 2 * n8).astype(np.int64)
    return masks8, (bits << np.arange(2 * n8, dtype=np.int64)).sum(-1)


def gemv_nm_fields(layer):
    """The interleaved decode pack of a non-2:4 layer re-laid out as (mask bytes
    [n_out, k/8], code fields [n_out, k/8]), plus every byte that no weight
    fills (rows padded to 16, k to 128) for a check that it is zero."""
    n_out, k, n, m = layer.n_out, layer.k, layer.n, layer.m
    n8 = 8 * n // m
    cb = (2 * n8 + 3) // 4 * 4
    has_mask = n8 < 8
    ub = (256 if has_mask else 0) + 32 * cb
    tiles, upr = (n_out + 15) // 16, (k + 127) // 128
    L = layer.layout()
    assert L.gemv_bytes == tiles * upr * ub
    raw = section(layer, "gemv", int(L.gemv_bytes)).reshape(tiles, upr, ub)
    rows, blocks = tiles * 16, upr * 16
    masks = np.full((rows, blocks), 0xFF, dtype=np.uint8)
    if has_mask:
        # [tile][unit][g][t][hi][s] -> row tile*16 + hi*8 + g, block unit*16 + t*4 + s
        mb = raw[:, :, :256].reshape(tiles, upr, 8, 4, 2, 4)
        masks = mb.transpose(0, 4, 2, 1, 3, 5).reshape(rows, blocks)
    cbytes = raw[:, :, 256 if has_mask else 0:].reshape(tiles, upr, 32, cb)
    cbits = np.unpackbits(cbytes, axis=-1, bitorder="little").astype(np.int64)  # [..., 32, cb*8]
    used = cbits[..., :16 * n8].reshape(tiles, upr, 8, 4, 2, 4, 2 * n8)  # g, t, hi, s, bit
    spare = cbits[..., 16 * n8:]
    fields = (used << np.arange(2 * n8, dtype=np.int64)).sum(-1)
    fields = fields.transpose(0, 4, 2, 1, 3, 5).reshape(rows, blocks)
    none = np.zeros(0, dtype=bool)
    pad = np.concatenate([masks[n_out:].ravel() != 0 if has_mask else none,
                          masks[:n_out, k // 8:].ravel() != 0 if has_mask else none,
                          fields[n_out:].ravel() != 0, fields[:n_out, k // 8:].ravel() != 0,
                          spare.ravel() != 0])
    return masks[:n_out, :k // 8], fields[:n_out, :k // 8], pad


def bf16_to_f64(t: torch.Tensor):
    return t.detach().float().cpu().numpy().astype(np.float64)
