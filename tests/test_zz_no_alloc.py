"""sbl_forward_noalloc: the forward pass for callers that cannot allocate.

Some callers cannot get device memory for a workspace (a plugin whose enqueue
hook must not allocate, a process whose device memory belongs to another
allocator, a loop that cannot afford cudaMalloc's implicit synchronisation).
For them the library keeps a fixed 16 MiB scratch array of its own.  These
tests call that entry point through the C ABI and check it against the
ordinary sbl_forward on the same inputs, on two calls in a row, so that the
second call runs on scratch that still holds the first call's contents.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_linear_layers_bitlinear_b200 import sbl, synth

RTOL, ATOL = 1e-3, 1e-2


def _close(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert (np.abs(gpu - ref) <= ATOL + RTOL * np.abs(ref)).all()


def test_noalloc_rejects_requests_beyond_its_scratch():
    # Returns before any CUDA call, so this part runs without a GPU.
    lib = sbl.lib()
    k = 2560
    layer = sbl.sbl_layer(256, k, 2, 4, 0, 0x1000)
    t_max = (sbl.NOALLOC_SCRATCH_BYTES - 65536) // k  # comfortably inside: codes + scales fit
    t_over = sbl.NOALLOC_SCRATCH_BYTES // k + 1
    dummy = ctypes.c_void_p(0x2000)
    assert lib.sbl_forward_noalloc(ctypes.byref(layer), dummy, t_over, dummy, None, None) == sbl.SBL_ERR_SCRATCH
    assert lib.sbl_forward_noalloc(ctypes.byref(layer), dummy, -1, dummy, None, None) == sbl.SBL_ERR_SHAPE
    assert lib.sbl_forward_noalloc(None, dummy, 4, dummy, None, None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_forward_noalloc(ctypes.byref(layer), None, 0, None, None, None) == sbl.SBL_OK
    assert t_max * k + 4 * t_max < sbl.NOALLOC_SCRATCH_BYTES
    # bad pointers are rejected before the scratch lookup touches a device
    assert lib.sbl_forward_noalloc(ctypes.byref(layer), None, 4, dummy, None, None) == sbl.SBL_ERR_INVALID_ARG
    assert lib.sbl_forward_noalloc(ctypes.byref(layer), ctypes.c_void_p(0x2008), 4, dummy, None, None) == \
        sbl.SBL_ERR_ALIGN
    assert lib.sbl_forward_noalloc(ctypes.byref(layer), dummy, 4, dummy, ctypes.c_void_p(0x3004), None) == \
        sbl.SBL_ERR_ALIGN
    unprepared = sbl.sbl_layer(256, k, 2, 4, 0, None)
    assert lib.sbl_forward_noalloc(ctypes.byref(unprepared), dummy, 4, dummy, None, None) == sbl.SBL_ERR_INVALID_ARG
    # the exact limit: k = 2048 and t = 8176 fill the 16 MiB to the byte
    # (codes, then the scales from the next 256-byte boundary)
    align256 = lambda v: (v + 255) // 256 * 256  # noqa: E731
    assert align256(8176 * 2048) + align256(8176 * 4) == sbl.NOALLOC_SCRATCH_BYTES
    wide = sbl.sbl_layer(256, 2048, 2, 4, 0, 0x1000)
    assert lib.sbl_forward_noalloc(ctypes.byref(wide), dummy, 8177, dummy, None, None) == sbl.SBL_ERR_SCRATCH


@pytest.mark.gpu
@pytest.mark.parametrize("n,m", [(2, 4), (6, 8)])
def test_noalloc_forward_matches_forward_on_two_calls(n, m):
    n_out, k = 392, 1024
    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, synth.master_weights(n_out, k, 31, device="cuda"))
    # The first call is the larger one, so the second runs over stale scratch.
    for call, t in enumerate((300, 77)):
        x = synth.activations(t, k, 40 + call, device="cuda")
        y_ref = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
        acc_ref = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
        ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
        sbl.forward(layer, x, t, y_ref, acc_debug=acc_ref, workspace=ws)

        y = torch.full((t, n_out), float("nan"), dtype=torch.float32, device="cuda")
        acc = torch.zeros((t, n_out), dtype=torch.int32, device="cuda")
        sbl.forward_noalloc(layer, x, t, y, acc)
        torch.cuda.synchronize()
        assert sbl.read_status(layer)[0] == sbl.SBL_OK

        assert torch.equal(acc, acc_ref)
        _close(y.cpu().numpy(), y_ref.cpu().numpy())
        assert torch.equal(y, y_ref)


def _compare_with_forward(layer, t, seed):
    """One sbl_forward_noalloc call against sbl_forward with a workspace on the
    same inputs: accumulators and y bit for bit."""
    k, n_out = layer.k, layer.n_out
    x = synth.activations(t, k, seed, device="cuda")
    y_ref = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc_ref = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, x, t, y_ref, acc_debug=acc_ref, workspace=ws)
    y = torch.full((t, n_out), float("nan"), dtype=torch.float32, device="cuda")
    acc = torch.zeros((t, n_out), dtype=torch.int32, device="cuda")
    sbl.forward_noalloc(layer, x, t, y, acc)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    assert torch.equal(acc, acc_ref)
    _close(y.cpu().numpy(), y_ref.cpu().numpy())
    assert torch.equal(y, y_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("n,m", [(2, 4), (6, 8)])
def test_noalloc_through_the_decode_kernel_over_stale_scratch(n, m):
    """A layer with the decode pack: a large call first fills the scratch,
    then decode-sized calls (the kernel quantises t <= 4 itself and writes the
    codes into the scratch; t = 16 runs the act-quant kernel into it first)."""
    n_out, k = 392, 1024
    layer = sbl.Layer.allocate(n_out, k, n, m, sbl.SBL_PACK_GEMV)
    sbl.prepare_weights(layer, synth.master_weights(n_out, k, 33, device="cuda"))
    for i, t in enumerate((300, 1, 4, 16)):
        assert sbl.forward_uses_gemv(layer, t) == (t <= 32)
        _compare_with_forward(layer, t, 50 + i)


@pytest.mark.gpu
def test_noalloc_at_its_exact_limit():
    """t = 8176 at k = 2048: codes and scales fill the 16 MiB to the byte, so
    the scales sit in its last 32 KB; one token more is refused."""
    n_out, k, t = 256, 2048, 8176
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, synth.master_weights(n_out, k, 34, device="cuda"))
    _compare_with_forward(layer, t, 60)
    x = torch.zeros((t + 1, k), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((t + 1, n_out), dtype=torch.float32, device="cuda")
    with pytest.raises(sbl.SblError):
        sbl.forward_noalloc(layer, x, t + 1, y)
