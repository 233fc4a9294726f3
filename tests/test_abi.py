"""C ABI checks that need no GPU: the library loads, exports every entry point
that include/sbl.h declares, and its host-only functions and argument
validation behave as documented (no compute is launched)."""
import ctypes
import os
import re
import subprocess

import pytest

from sparse_linear_layers_bitlinear_b200 import build, sbl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sbl.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return sbl.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sbl_[a-z0-9_]+)\s*\(", text)))


class _FakeBlob:
    """Stands in for a device blob: only its (aligned) address is read."""

    def data_ptr(self):
        return 0x10000


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for required in ("sbl_prepare_weights", "sbl_forward", "sbl_backward", "sbl_prepared_bytes",
                     "sbl_workspace_bytes", "sbl_read_status"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", sbl.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (sbl_[a-z0-9_]+)$", out.stdout, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)
    assert set(names) == set(sbl.SIGNATURES), "binding and header disagree"


def test_version(lib):
    assert "sm_100a" in sbl.version()


def test_layout_sections_are_aligned_and_disjoint(lib):
    g = sbl.SBL_PACK_GEMV
    g6 = g | sbl.SBL_PACK_GEMV_6BIT
    for (n_out, k, n, m, flags) in [(6912, 2560, 2, 4, 0), (2560, 6912, 6, 8, 0), (264, 320, 2, 4, g),
                                    (8, 64, 1, 2, 0), (2560, 6912, 6, 8, g), (264, 320, 3, 8, g), (8, 64, 1, 2, g),
                                    (136, 448, 8, 8, g), (264, 320, 2, 4, g6), (6912, 2560, 2, 4, g6)]:
        L = sbl.prepared_layout(n_out, k, n, m, flags)
        spans = [("header", L.header, 4096), ("scratch", L.scratch, 1024 * 40 * 8 + 1024 * 32 + 256), ("mask", L.mask, n_out * k // m), ("weff_bf16", L.weff_bf16, 2 * n_out * k)]
        if (n, m) == (2, 4):
            spans += [("sp_values", L.sp_values, n_out * k // 2), ("sp_meta", L.sp_meta, L.sp_meta_bytes)]
            assert L.sp_meta_bytes == ((n_out + 255) // 256 * 256) * ((k + 255) // 256 * 256) // 8
            assert L.codes == 0
            if flags & sbl.SBL_PACK_GEMV:  # interleaved units: a byte or 6 bits a group of four
                unit = 384 if flags & sbl.SBL_PACK_GEMV_6BIT else 512
                assert L.gemv_bytes == ((n_out + 15) // 16) * ((k + 127) // 128) * unit
        else:
            spans.append(("codes", L.codes, n_out * k))
            assert L.sp_values == 0 and L.sp_meta == 0
            if flags & sbl.SBL_PACK_GEMV:
                # units of 16 rows x 128 k: a 256-byte mask block (n < m) and 32 lanes' code bytes
                n8 = 8 * n // m
                unit = (256 if n8 < 8 else 0) + 32 * ((2 * n8 + 3) // 4 * 4)
                assert L.gemv_bytes == ((n_out + 15) // 16) * ((k + 127) // 128) * unit
        if flags & sbl.SBL_PACK_GEMV:
            spans.append(("gemv", L.gemv, L.gemv_bytes))
        else:
            assert L.gemv == 0 and L.gemv_bytes == 0
        spans.sort(key=lambda s: s[1])
        for (_, off, size), (_, nxt, _) in zip(spans, spans[1:]):
            assert off % 256 == 0 and off + size <= nxt
        assert spans[-1][1] + spans[-1][2] <= L.total_bytes
        assert sbl.prepared_bytes(n_out, k, n, m, flags) == L.total_bytes
        assert L.header <= L.gamma < L.header + 4096 and L.g == L.gamma + 4


def test_ablation_flags_are_accepted_and_unknown_bits_rejected(lib):
    base = sbl.prepared_bytes(264, 320, 2, 4, 0)
    assert sbl.prepared_bytes(264, 320, 2, 4, sbl.SBL_MASK_FROM_QUANT) == base  # same sections
    assert sbl.prepared_bytes(264, 320, 6, 8, sbl.SBL_MASK_FROM_QUANT) > 0
    assert sbl.prepared_bytes(264, 320, 2, 4, sbl.SBL_MASK_FROM_QUANT | sbl.SBL_PACK_GEMV) > base
    assert sbl.prepared_bytes(264, 320, 2, 4, 1 << 5) == 0
    with pytest.raises(sbl.SblError):
        sbl.prepared_layout(264, 320, 2, 4, 1 << 5)


def test_forward_dispatch_query(lib):
    def uses(n_out, k, n, m, flags, t):
        return sbl.forward_uses_gemv(sbl.Layer(n_out, k, n, m, flags, _FakeBlob()), t)

    g = sbl.SBL_PACK_GEMV
    for t in (1, 4, 8, 16, 32):
        assert uses(6912, 2560, 2, 4, g, t) and uses(2560, 2560, 2, 4, g, t)
        assert uses(2560, 6912, 6, 8, g, t) == (t <= 16)  # 32 token rows of k = 6912 exceed shared memory
        assert uses(2560, 2560, 4, 8, g, t) and uses(2560, 2560, 8, 8, g, t)
    assert not uses(256, 256, 2, 4, g, 33)      # beyond the decode kernel's token count
    assert not uses(6912, 2560, 2, 4, 0, 1)     # no decode pack
    assert not uses(2560, 6912, 6, 8, 0, 1)
    assert not uses(6912, 2560, 2, 4, g, 0)
    assert not uses(6912, 2560, 6, 4, g, 1)     # not a valid layer
    g6 = g | sbl.SBL_PACK_GEMV_6BIT
    for t in (1, 4, 16, 32):
        # its 4 KB table (against 16 KB for the byte pack) leaves room for 32 rows of k = 6912
        assert uses(6912, 2560, 2, 4, g6, t) and uses(2560, 6912, 2, 4, g6, t)
        assert uses(2560, 6912, 2, 4, g, t) == (t <= 16)
    assert not uses(6912, 2560, 2, 4, g6, 33)
    assert not uses(2560, 2560, 6, 8, g6, 1)     # the 6-bit code is a 2:4 pack only


def test_backward_workspace_for_the_quantised_x_operand(lib):
    q = sbl.SBL_DW_QUANT_X
    assert sbl.backward_workspace_bytes(40, 256, 0) == 0
    assert sbl.backward_workspace_bytes(40, 256, q) == 40 * 256 * 2
    assert sbl.backward_workspace_bytes(40, 256, q | sbl.SBL_NO_DW) == 0  # no dW, no operand
    assert sbl.backward_workspace_bytes(0, 256, q) == 0
    # rejected before anything touches a device
    layer = sbl.sbl_layer(256, 256, 2, 4, 0, 0x1000)
    p = ctypes.c_void_p
    args = (ctypes.byref(layer), p(0x2000), p(0x3000), 4, p(0x4000), p(0x5000))
    assert lib.sbl_backward(*args, q, None) == sbl.SBL_ERR_INVALID_ARG          # needs a workspace
    assert lib.sbl_backward_ws(*args, q, None, None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_backward_ws(*args, q, p(0x6008), None) == sbl.SBL_ERR_ALIGN
    assert lib.sbl_backward_ws(*args, q | (1 << 6), p(0x6000), None) == sbl.SBL_ERR_INVALID_ARG


@pytest.mark.parametrize("args,code", [
    ((256, 256, 2, 3, 0), sbl.SBL_ERR_UNSUPPORTED_NM),
    ((256, 256, 0, 4, 0), sbl.SBL_ERR_UNSUPPORTED_NM),
    ((256, 256, 5, 4, 0), sbl.SBL_ERR_UNSUPPORTED_NM),
    ((256, 256, 6, 4, sbl.SBL_PACK_GEMV), sbl.SBL_ERR_UNSUPPORTED_NM),
    ((256, 96, 2, 4, 0), sbl.SBL_ERR_SHAPE),
    ((250, 256, 2, 4, 0), sbl.SBL_ERR_SHAPE),
    ((0, 256, 2, 4, 0), sbl.SBL_ERR_SHAPE),
    ((256, 256, 2, 4, 1 << 9), sbl.SBL_ERR_INVALID_ARG),
    ((256, 256, 2, 4, sbl.SBL_PACK_GEMV_6BIT), sbl.SBL_ERR_INVALID_ARG),  # needs the decode pack
    ((256, 256, 6, 8, sbl.SBL_PACK_GEMV | sbl.SBL_PACK_GEMV_6BIT), sbl.SBL_ERR_UNSUPPORTED_NM),
    ((256, 256, 4, 8, sbl.SBL_PACK_GEMV | sbl.SBL_PACK_GEMV_6BIT), sbl.SBL_ERR_UNSUPPORTED_NM),
])
def test_layout_rejects_bad_arguments(lib, args, code):
    out = sbl.sbl_blob_layout()
    assert lib.sbl_prepared_layout(*args, ctypes.byref(out)) == code
    assert sbl.prepared_bytes(*args) == 0


def test_workspace_bytes(lib):
    # codes, scales, then one counter per 16 tokens, each piece 256-byte aligned
    assert sbl.workspace_bytes(4096, 2560) == 4096 * 2560 + 4096 * 4 + 1024
    assert sbl.workspace_bytes(3, 64) == 256 + 256 + 256
    assert sbl.workspace_bytes(300, 64) == 19200 + 1280 + 256
    assert sbl.workspace_bytes(0, 64) == 0


def test_entry_points_validate_before_touching_the_device(lib):
    # These return before any CUDA call, so they run on a machine without a GPU.
    launched_before = sbl.launch_count()
    layer = sbl.sbl_layer(256, 256, 2, 4, 0, 0x1000)
    assert lib.sbl_prepare_weights(None, ctypes.c_void_p(0x2000), None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_prepare_weights(ctypes.byref(layer), None, None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_prepare_weights(ctypes.byref(layer), ctypes.c_void_p(0x2001), None) == sbl.SBL_ERR_ALIGN
    misaligned = sbl.sbl_layer(256, 256, 2, 4, 0, 0x1010)
    assert lib.sbl_prepare_weights(ctypes.byref(misaligned), ctypes.c_void_p(0x2000), None) == sbl.SBL_ERR_ALIGN
    bad_nm = sbl.sbl_layer(256, 256, 3, 2, 0, 0x1000)
    assert lib.sbl_prepare_weights(ctypes.byref(bad_nm), ctypes.c_void_p(0x2000), None) == sbl.SBL_ERR_UNSUPPORTED_NM
    assert lib.sbl_forward(ctypes.byref(layer), None, -1, None, None, None, None, None, None) == sbl.SBL_ERR_SHAPE
    assert lib.sbl_forward(ctypes.byref(layer), None, 0, None, None, None, None, None, None) == sbl.SBL_OK
    assert lib.sbl_forward(ctypes.byref(layer), None, 8, None, None, None, None, None, None) == sbl.SBL_ERR_INVALID_ARG
    # no workspace and no explicit xq / scale buffers
    assert lib.sbl_forward(ctypes.byref(layer), ctypes.c_void_p(0x3000), 8, ctypes.c_void_p(0x4000), None, None, None,
                           None, None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_backward(ctypes.byref(layer), None, None, 4, None, None, 0, None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_backward(ctypes.byref(layer), None, None, 4, None, None, 1 << 7, None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_selftest_wait_timeout(None, 1000, None) == sbl.SBL_ERR_INVALID_ARG
    q = lib.sbl_quantize_activations
    P = ctypes.c_void_p
    assert q(P(0x1000), 4, 100, P(0x2000), P(0x3000), P(0x4000), None) == sbl.SBL_ERR_SHAPE
    assert q(P(0x1000), -1, 128, P(0x2000), P(0x3000), P(0x4000), None) == sbl.SBL_ERR_SHAPE
    assert q(None, 0, 128, None, None, None, None) == sbl.SBL_OK
    assert q(P(0x1000), 4, 128, P(0x2000), P(0x3000), None, None) == sbl.SBL_ERR_INVALID_ARG
    assert q(P(0x1008), 4, 128, P(0x2000), P(0x3000), P(0x4000), None) == sbl.SBL_ERR_ALIGN
    assert q(P(0x1000), 4, 128, P(0x2000), P(0x3000), P(0x4002), None) == sbl.SBL_ERR_ALIGN
    st = ctypes.c_void_p(0x5000)
    for kind, stages, pairs, status in ((3, 16, 1, st), (-1, 16, 1, st), (0, 0, 1, st), (0, (1 << 20) + 1, 1, st),
                                        (0, 16, 0, st), (0, 16, 1, None)):
        assert lib.sbl_selftest_mma_rate(kind, stages, pairs, status, None, None) == sbl.SBL_ERR_INVALID_ARG
    p = ctypes.c_void_p
    assert lib.sbl_forward_quantized(ctypes.byref(layer), None, p(0x3000), 8, p(0x4000), None, None) == \
        sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_forward_quantized(ctypes.byref(layer), p(0x2000), p(0x3008), 8, p(0x4000), None, None) == \
        sbl.SBL_ERR_ALIGN
    assert lib.sbl_forward_quantized(ctypes.byref(layer), None, None, 0, None, None, None) == sbl.SBL_OK
    assert lib.sbl_forward_quantized(ctypes.byref(layer), None, None, -1, None, None, None) == sbl.SBL_ERR_SHAPE
    # rejected calls enqueue nothing, so they launch nothing
    assert sbl.launch_count() == launched_before


def test_grouped_prepare_validates_before_touching_the_device(lib):
    launched = sbl.launch_count()
    p = ctypes.c_void_p
    L = lambda n, m, blob: sbl.sbl_layer(256, 256, n, m, 0, blob)  # noqa: E731

    def call(layers, masters, count=None):
        arr = (sbl.sbl_layer * len(layers))(*layers)
        ws = (ctypes.c_void_p * len(masters))(*masters)
        return lib.sbl_prepare_weights_grouped(arr, ws, len(layers) if count is None else count, None)

    two = [L(2, 4, 0x1000), L(1, 4, 0x2000)]
    assert call(two, [0x10000, 0x20000], count=0) == sbl.SBL_ERR_INVALID_ARG
    assert call(two, [0x10000, 0x20000], count=9) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_prepare_weights_grouped(None, None, 1, None) == sbl.SBL_ERR_INVALID_ARG
    assert call([L(2, 4, 0x1000), L(6, 8, 0x2000)], [0x10000, 0x20000]) == sbl.SBL_ERR_UNSUPPORTED_NM
    assert call([L(2, 4, 0x1000), L(1, 4, 0x1000)], [0x10000, 0x20000]) == sbl.SBL_ERR_INVALID_ARG  # one blob
    assert call(two, [0x10000, None]) == sbl.SBL_ERR_INVALID_ARG
    assert call(two, [0x10000, 0x20008]) == sbl.SBL_ERR_ALIGN
    assert call([L(2, 4, 0x1000), L(1, 4, 0x2010)], [0x10000, 0x20000]) == sbl.SBL_ERR_ALIGN  # blob alignment
    assert sbl.launch_count() == launched
