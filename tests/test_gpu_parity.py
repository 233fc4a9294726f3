"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integer, byte and index results (gamma bits, masks, codes, packed forms,
int8 activations, int32 accumulators) must match bit for bit; y (fp32) is
checked bit for bit too and, as the stated bound, within rel 1e-3 / abs 1e-2;
gradients within rel 1e-3 / abs 1e-2 (fp32 mode) or one bf16 step plus abs
1e-2 (bf16 mode) of the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_linear_layers_bitlinear_b200 import sbl, synth
from tests import blob_decode as bd

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-3, 1e-2
BF16_REL = 2.0 ** -7  # one bf16 step, relative


def _dev(t):
    return t.to("cuda")


def _close(gpu, ref, rtol=RTOL, atol=ATOL):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tolerance; worst err {err.max()}"


def _check_prepared(layer, w, n, m):
    ref = oracle.prepare(w, n, m, mask_from_codes=bool(layer.flags & sbl.SBL_MASK_FROM_QUANT))
    gamma, g, status = bd.header_scalars(layer)
    assert status == 0
    assert np.float32(gamma).view(np.uint32) == np.float32(ref["gamma"]).view(np.uint32)
    assert np.float32(g).view(np.uint32) == np.float32(ref["g"]).view(np.uint32)
    assert np.array_equal(bd.mask(layer), ref["mask"])
    assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"])
    if (n, m) == (2, 4):
        vals, meta = oracle.pack24(ref["weff"], ref["mask"])
        assert np.array_equal(bd.sp_values(layer), vals)
        canon, pad_rows, pad_cols = bd.sp_meta_canonical(layer)
        assert np.array_equal(canon, meta)
        assert (pad_rows == 0x44).all() and (pad_cols == 0x44).all()
        if layer.flags & sbl.SBL_PACK_GEMV_6BIT:
            got, pad = bd.gemv_code6(layer)
            assert not pad.any(), "bytes outside the matrix must be zero"
            assert np.array_equal(got, oracle.pack24_code6(ref["weff"], ref["mask"]))
        elif layer.flags & sbl.SBL_PACK_GEMV:
            gb, pad = bd.gemv_bytes(layer)
            assert not pad.any(), "bytes outside the matrix must be zero"
            nib, c0, c1 = bd.decode_gemv(gb)
            mnib = np.stack([meta & 0xF, meta >> 4], axis=-1).reshape(meta.shape[0], -1)
            assert np.array_equal(nib, mnib)
            assert np.array_equal(c0, vals[:, 0::2]) and np.array_equal(c1, vals[:, 1::2])
    else:
        assert np.array_equal(bd.codes(layer), ref["weff"])
        if layer.flags & sbl.SBL_PACK_GEMV:
            masks8, codes = oracle.pack_nm(ref["weff"], ref["mask"], n, m)
            want_m, want_f = bd.nm_pack_fields(masks8, codes, n, m)
            got_m, got_f, pad = bd.gemv_nm_fields(layer)
            if n < m:
                assert np.array_equal(got_m, want_m)
            assert np.array_equal(got_f, want_f)
            assert not pad.any(), "bytes outside the matrix must be zero"
    return ref


CASES = [
    # n_out, k, n, m, t
    (256, 256, 2, 4, 16),     # the small single-forward workload
    (264, 320, 2, 4, 300),    # ragged rows, k not a multiple of 128, ragged tokens
    (136, 448, 6, 8, 77),
    (128, 384, 4, 8, 129),
    (520, 192, 1, 4, 33),
    (64, 64, 3, 4, 3),
    (8, 64, 2, 4, 5),
    (384, 512, 8, 8, 260),    # N = M: plain ternary BitLinear
    (200, 128, 1, 2, 50),
    (392, 832, 3, 8, 513),
]


@pytest.mark.parametrize("n_out,k,n,m,t", CASES)
def test_prepare_forward_backward_parity(n_out, k, n, m, t):
    seed = n_out * 7 + k + 13 * n + m
    w = synth.master_weights(n_out, k, seed)
    x = synth.activations(t, k, seed + 1)
    dy = synth.upstream_grad(t, n_out, seed + 2)

    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, _dev(w))
    torch.cuda.synchronize()
    ref = _check_prepared(layer, w, n, m)

    xd, dyd = _dev(x), _dev(dy)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    sbl.forward(layer, xd, t, y, xq, ap, acc)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK

    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    acc_ref = oracle.gemm_acc(xq_ref, ref["weff"])
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    y_ref = oracle.dequant(acc_ref, ap_ref, ref["g"])
    y_gpu = y.cpu().numpy()
    _close(y_gpu, y_ref)
    assert np.array_equal(y_gpu.view(np.uint32), y_ref.view(np.uint32))

    # backward, fp32 outputs
    dx = torch.empty((t, k), dtype=torch.float32, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.float32, device="cuda")
    sbl.backward(layer, xd, dyd, t, dx, dw, sbl.SBL_GRAD_F32)
    torch.cuda.synchronize()
    dx_ref = oracle.grad_x(dy, ref["weff"], ref["g"])
    dw_ref = oracle.grad_w(dy, x)
    _close(dx.cpu().numpy(), dx_ref)
    _close(dw.cpu().numpy(), dw_ref)

    # backward, bf16 outputs: within one bf16 step of the rounded oracle
    dx16 = torch.empty((t, k), dtype=torch.bfloat16, device="cuda")
    dw16 = torch.empty((n_out, k), dtype=torch.bfloat16, device="cuda")
    sbl.backward(layer, xd, dyd, t, dx16, dw16, 0)
    torch.cuda.synchronize()
    _close(bd.bf16_to_f64(dx16), dx_ref, rtol=BF16_REL, atol=ATOL)
    _close(bd.bf16_to_f64(dw16), dw_ref, rtol=BF16_REL, atol=ATOL)
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


@pytest.mark.parametrize("t", [1, 2, 3, 4, 5, 7, 8, 9, 16, 17, 24, 32])
def test_gemv_path_parity(t):
    n_out, k = 392, 640
    w = synth.master_weights(n_out, k, 3)
    x = synth.activations(t, k, 4)
    layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_PACK_GEMV)
    sbl.prepare_weights(layer, _dev(w))
    torch.cuda.synchronize()
    ref = _check_prepared(layer, w, 2, 4)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap, acc)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    acc_ref = oracle.gemm_acc(xq_ref, ref["weff"])
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    y_ref = oracle.dequant(acc_ref, ap_ref, ref["g"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), y_ref.view(np.uint32))


def test_workspace_path_matches_explicit_buffers():
    n_out, k, t = 256, 512, 40
    w = synth.master_weights(n_out, k, 8)
    x = _dev(synth.activations(t, k, 9))
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(w))
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    y1 = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    sbl.forward(layer, x, t, y1, workspace=ws)
    y2 = torch.empty_like(y1)
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, x, t, y2, xq, ap)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_empty_batch():
    n_out, k = 64, 128
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 1)))
    y = torch.empty((0, n_out), dtype=torch.float32, device="cuda")
    sbl.forward(layer, None, 0, y)
    dw = torch.full((n_out, k), 7.0, dtype=torch.float32, device="cuda")
    sbl.backward(layer, None, None, 0, None, dw, sbl.SBL_GRAD_F32 | sbl.SBL_NO_DX)
    torch.cuda.synchronize()
    assert (dw == 0).all()


def test_nonfinite_inputs_raise_status():
    n_out, k = 64, 128
    w = synth.master_weights(n_out, k, 2)
    w[3, 5] = float("nan")
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(w))
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_ERR_NONFINITE and bits & sbl.SBL_STATUS_NONFINITE_W
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 2)))
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    x = synth.activations(4, k, 3)
    x[1, 7] = float("inf")
    y = torch.empty((4, n_out), dtype=torch.float32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(4, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, _dev(x), 4, y, workspace=ws)
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_ERR_NONFINITE and bits & sbl.SBL_STATUS_NONFINITE_X
    sbl.clear_status(layer)
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


def test_bounded_wait_reports_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sbl.selftest_wait_timeout(status, 2_000_000)  # 2 ms on a barrier nothing arrives on
    torch.cuda.synchronize()
    assert int(status.item()) & sbl.SBL_STATUS_TIMEOUT
    # the context is still usable afterwards
    assert float(torch.ones(4, device="cuda").sum()) == 4.0


@pytest.mark.parametrize("kind,macs", [(0, 256 * 240 * 256), (1, 256 * 256 * 128), (2, 256 * 256 * 64)])
def test_mma_rate_selftest_runs_and_drains(kind, macs):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    assert sbl.selftest_mma_rate(kind, 64, pairs, status) == macs
    assert sbl.selftest_mma_rate(kind, 1, 1, status) == macs
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    with pytest.raises(sbl.SblError):
        sbl.selftest_mma_rate(kind, 64, pairs + 1, status)


def test_gamma_scale_readback():
    w = synth.master_weights(128, 256, 5)
    layer = sbl.Layer.allocate(128, 256, 6, 8)
    sbl.prepare_weights(layer, _dev(w))
    gamma, g = sbl.read_scale(layer)
    assert np.float32(gamma) == oracle.absmean_gamma(w)
    assert np.float32(g) == oracle.clamped_scale(oracle.absmean_gamma(w))


@pytest.mark.parametrize("kind", ["bf16_subnormal", "all_exponents", "near_max", "constant", "gauss_few_tiny"])
def test_gamma_and_codes_at_extreme_magnitudes(kind):
    """The exact absmean over inputs that reach the corners of the bf16 range:
    subnormal masters (gamma lands in the fp32 subnormal range or rounds to 0),
    magnitudes spread over every finite exponent (every partial-sum bin in
    use), magnitudes near the bf16 maximum, and a constant magnitude."""
    n_out, k, n, m = 136, 320, 2, 4
    rng = np.random.default_rng({"bf16_subnormal": 1, "all_exponents": 2, "near_max": 3, "constant": 4,
                                 "gauss_few_tiny": 5}[kind])
    size = (n_out, k)
    if kind == "bf16_subnormal":
        mag = rng.integers(0, 0x80, size=size)
    elif kind == "all_exponents":
        mag = rng.integers(0, 0x7F80, size=size)
    elif kind == "near_max":
        mag = rng.integers(0x7E00, 0x7F80, size=size)
    elif kind == "constant":
        mag = np.full(size, 0x3C00)
    else:  # Gaussian masters with a few subnormal and tiny ones mixed in
        mag = synth.bits(synth.master_weights(n_out, k, 77)).astype(np.int64) & 0x7FFF
        idx = rng.integers(0, mag.size, size=40)
        mag.ravel()[idx[:20]] = rng.integers(1, 0x80, size=20)
        mag.ravel()[idx[20:]] = rng.integers(0x0800, 0x1000, size=20)
    sign = rng.integers(0, 2, size=size) << 15
    bits = (mag | sign).astype(np.uint16)
    w = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, _dev(w))
    torch.cuda.synchronize()
    _check_prepared(layer, w, n, m)


@pytest.mark.parametrize("n_out,k,n,m,t", [(264, 320, 2, 4, 70), (136, 448, 6, 8, 33), (200, 128, 1, 2, 9),
                                           (128, 384, 4, 8, 17)])
def test_ablation_mask_from_codes(n_out, k, n, m, t):
    """The pages' ablation that builds the mask from the ternary codes: the
    prepared sections and the forward match the oracle's code-based mask."""
    seed = 4 * n_out + k + n
    w = synth.master_weights(n_out, k, seed)
    x = synth.activations(t, k, seed + 1)
    layer = sbl.Layer.allocate(n_out, k, n, m, sbl.SBL_MASK_FROM_QUANT)
    sbl.prepare_weights(layer, _dev(w))
    torch.cuda.synchronize()
    ref = oracle.prepare(w, n, m, mask_from_codes=True)
    gamma, g, status = bd.header_scalars(layer)
    assert status == 0 and np.float32(g) == ref["g"]
    assert np.array_equal(bd.mask(layer), ref["mask"])
    assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"])
    if (n, m) == (2, 4):
        vals, meta = oracle.pack24(ref["weff"], ref["mask"])
        assert np.array_equal(bd.sp_values(layer), vals)
        assert np.array_equal(bd.sp_meta_canonical(layer)[0], meta)
    else:
        assert np.array_equal(bd.codes(layer), ref["weff"])
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap, acc)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    acc_ref = oracle.gemm_acc(xq_ref, ref["weff"])
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert np.array_equal(y.cpu().numpy().view(np.uint32), oracle.dequant(acc_ref, ap_ref, ref["g"]).view(np.uint32))


@pytest.mark.parametrize("n_out,k,n,m,t", [(264, 320, 2, 4, 70), (136, 448, 6, 8, 33), (200, 128, 1, 2, 9),
                                           (392, 832, 3, 8, 130)])
@pytest.mark.parametrize("only_dw", [False, True])
def test_ablation_masked_grad(n_out, k, n, m, t, only_dw):
    """The pages' blocked-gradient ablation: dW is the dense dY^T X on kept
    positions and exactly 0 on pruned ones; dX is unchanged."""
    seed = 3 * n_out + k + m
    w = synth.master_weights(n_out, k, seed)
    x = synth.activations(t, k, seed + 1)
    dy = synth.upstream_grad(t, n_out, seed + 2)
    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, _dev(w))
    ref = oracle.prepare(w, n, m)
    dw_ref = oracle.grad_w_masked(dy, x, ref["mask"], m)
    flags = sbl.SBL_MASKED_GRAD | (sbl.SBL_NO_DX if only_dw else 0)
    dx = None if only_dw else torch.empty((t, k), dtype=torch.float32, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.float32, device="cuda")
    sbl.backward(layer, _dev(x), _dev(dy), t, dx, dw, flags | sbl.SBL_GRAD_F32)
    torch.cuda.synchronize()
    dw_gpu = dw.cpu().numpy()
    _close(dw_gpu, dw_ref)
    assert (dw_gpu[dw_ref == 0] == 0).all() and np.count_nonzero(dw_gpu) <= n_out * k * n // m
    if not only_dw:
        _close(dx.cpu().numpy(), oracle.grad_x(dy, ref["weff"], ref["g"]))
    # bf16 outputs, the same launch shape (one dual launch, or dW alone)
    dx16 = None if only_dw else torch.empty((t, k), dtype=torch.bfloat16, device="cuda")
    dw16 = torch.empty((n_out, k), dtype=torch.bfloat16, device="cuda")
    sbl.backward(layer, _dev(x), _dev(dy), t, dx16, dw16, flags)
    torch.cuda.synchronize()
    _close(bd.bf16_to_f64(dw16), dw_ref, rtol=BF16_REL, atol=ATOL)
    assert (bd.bf16_to_f64(dw16)[dw_ref == 0] == 0).all()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


def test_dense_to_sparse_switch():
    """The schedule the pages compare against sparse-from-scratch ([de] §4):
    the same masters run dense ternary (N = M) first and then 2:4 and 6:8.
    Each pattern is its own prepared layer; switching is preparing the masters
    into the other one, and every stage matches the oracle."""
    n_out, k, t = 264, 384, 40
    w = synth.master_weights(n_out, k, 91)
    x = synth.activations(t, k, 92)
    xq_ref, ap_ref = oracle.act_quant(x)
    for n, m in [(4, 4), (8, 8), (2, 4), (6, 8)]:
        layer = sbl.Layer.allocate(n_out, k, n, m)
        sbl.prepare_weights(layer, _dev(w))
        ref = _check_prepared(layer, w, n, m)
        y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
        acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
        ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
        sbl.forward(layer, _dev(x), t, y, acc_debug=acc, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(acc.cpu().numpy(), oracle.gemm_acc(xq_ref, ref["weff"]))
        if n == m:  # dense ternary: nothing pruned
            assert (bd.mask(layer) == (1 << m) - 1).all()


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8)])
def test_maximum_row_length(n, m):
    """k at the library's limit (131072: |acc| <= 127 k stays exactly
    representable in fp32): prepare, the long-row activation quantiser, the
    forward GEMM over 512 k blocks and both backward products."""
    n_out, k, t = 16, 131072, 5
    w = synth.master_weights(n_out, k, 71)
    x = synth.activations(t, k, 72)
    dy = synth.upstream_grad(t, n_out, 73)
    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, _dev(w))
    torch.cuda.synchronize()
    ref = _check_prepared(layer, w, n, m)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap, acc)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    acc_ref = oracle.gemm_acc(xq_ref, ref["weff"])
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert np.array_equal(y.cpu().numpy().view(np.uint32), oracle.dequant(acc_ref, ap_ref, ref["g"]).view(np.uint32))
    dx = torch.empty((t, k), dtype=torch.float32, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.float32, device="cuda")
    sbl.backward(layer, _dev(x), _dev(dy), t, dx, dw, sbl.SBL_GRAD_F32)
    torch.cuda.synchronize()
    _close(dx.cpu().numpy(), oracle.grad_x(dy, ref["weff"], ref["g"]))
    _close(dw.cpu().numpy(), oracle.grad_w(dy, x))
    with pytest.raises(sbl.SblError):  # one step beyond the limit is refused before anything runs
        sbl.Layer.allocate(n_out, k + 64, n, m)


def test_degenerate_all_zero_inputs():
    """All-zero masters give gamma = 0, so g = 1e-5 and every code 0; all-zero
    activations give a' = 1e-5 and zero codes; all-zero upstream gradients
    give zero gradients.  Every output is exactly 0 and no error is raised."""
    n_out, k, t = 264, 320, 33
    for n, m in [(2, 4), (6, 8)]:
        w = torch.zeros((n_out, k), dtype=torch.bfloat16)
        x = torch.zeros((t, k), dtype=torch.bfloat16)
        dy = torch.zeros((t, n_out), dtype=torch.bfloat16)
        layer = sbl.Layer.allocate(n_out, k, n, m)
        sbl.prepare_weights(layer, _dev(w))
        torch.cuda.synchronize()
        ref = _check_prepared(layer, w, n, m)
        gamma, g, _ = bd.header_scalars(layer)
        assert gamma == 0.0 and np.float32(g) == np.float32(1e-5)
        assert not ref["weff"].any()
        assert (bd.mask(layer) == oracle.nm_mask(synth.bits(w), n, m)).all()  # all ties: lowest indices
        y = torch.full((t, n_out), 7.0, dtype=torch.float32, device="cuda")
        xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
        ap = torch.empty((t,), dtype=torch.float32, device="cuda")
        sbl.forward(layer, _dev(x), t, y, xq, ap)
        dx = torch.full((t, k), 7.0, dtype=torch.float32, device="cuda")
        dw = torch.full((n_out, k), 7.0, dtype=torch.float32, device="cuda")
        sbl.backward(layer, _dev(x), _dev(dy), t, dx, dw, sbl.SBL_GRAD_F32)
        torch.cuda.synchronize()
        assert (y == 0).all() and (xq == 0).all() and (dx == 0).all() and (dw == 0).all()
        assert np.array_equal(ap.cpu().numpy(), np.full(t, np.float32(1e-5)))
        assert sbl.read_status(layer)[0] == sbl.SBL_OK


@pytest.mark.parametrize("fill", ["random", "ones", "zeros"])
def test_prepare_on_uninitialised_blob_and_repeats(fill):
    """The prepare kernel's grid barrier keeps its state in the blob's scratch
    and needs no initialisation: a blob holding arbitrary bytes prepares
    correctly, and so does every later prepare of the same blob."""
    n_out, k, n, m = 520, 1024, 2, 4
    layer = sbl.Layer.allocate(n_out, k, n, m)
    if fill == "random":
        gen = torch.Generator().manual_seed(11)
        layer.blob.copy_(torch.randint(0, 256, layer.blob.shape, dtype=torch.uint8, generator=gen))
    elif fill == "ones":
        layer.blob.fill_(0xFF)
    else:
        layer.blob.zero_()
    for rep in range(3):
        w = synth.master_weights(n_out, k, 100 + rep)
        sbl.prepare_weights(layer, _dev(w))
        torch.cuda.synchronize()
        _check_prepared(layer, w, n, m)


@pytest.mark.parametrize("k", [64, 768, 1088, 2048, 2560, 3072, 3136, 4160, 6912, 12352, 16384, 16448])
def test_act_quant_row_lengths(k):
    """Activation codes and scales for row lengths that exercise every
    register-resident variant of the act-quant kernel and its long-row path."""
    n_out, t = 8, 5
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 50)))
    x = synth.activations(t, k, 51)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))


def test_launch_count_per_step():
    """The library's own launch counter: one prepare, two forward kernels
    (act-quant, 2:4 GEMM) and one backward launch per training step."""
    n_out, k, t = 512, 768, 320
    w = synth.master_weights(n_out, k, 71, device="cuda")
    x = synth.activations(t, k, 72, device="cuda")
    dy = synth.upstream_grad(t, n_out, 73, device="cuda")
    layer = sbl.Layer.allocate(n_out, k, 2, 4, device="cuda")
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    dx = torch.empty((t, k), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.bfloat16, device="cuda")
    c0 = sbl.launch_count()
    sbl.prepare_weights(layer, w)
    c1 = sbl.launch_count()
    sbl.forward(layer, x, t, y, workspace=ws)
    c2 = sbl.launch_count()
    sbl.backward(layer, x, dy, t, dx, dw, 0)
    c3 = sbl.launch_count()
    sbl.forward(layer, x, 0, y, workspace=ws)  # empty batch: nothing to launch
    c4 = sbl.launch_count()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    assert (c1 - c0, c2 - c1, c3 - c2, c4 - c3) == (1, 2, 1, 0)


@pytest.mark.parametrize("n_out,k,n,m,t", [(264, 320, 2, 4, 70), (136, 448, 6, 8, 33), (392, 832, 3, 8, 130)])
@pytest.mark.parametrize("only_dw", [False, True])
def test_dw_quant_x(n_out, k, n, m, t, only_dw):
    """The detach-form reading of the STE for the quantiser: dW is taken
    against xhat = RN_bf16(xq a' / 127), which the call leaves in its
    workspace (bit-exact against the oracle); dX is the same as without it."""
    seed = 5 * n_out + k + m
    w = synth.master_weights(n_out, k, seed)
    x = synth.activations(t, k, seed + 1)
    dy = synth.upstream_grad(t, n_out, seed + 2)
    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, _dev(w))
    ref = oracle.prepare(w, n, m)
    xq_ref, ap_ref = oracle.act_quant(x)
    xhat_ref = oracle.dequant_act(xq_ref, ap_ref)
    dw_ref = oracle.grad_w_quant_x(dy, x)
    flags = sbl.SBL_DW_QUANT_X | (sbl.SBL_NO_DX if only_dw else 0)
    nbytes = sbl.backward_workspace_bytes(t, k, flags)
    assert nbytes == t * k * 2
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device="cuda")
    with pytest.raises(sbl.SblError):
        sbl.backward(layer, _dev(x), _dev(dy), t, None, None, flags)  # no workspace
    for f32 in (True, False):
        dt = torch.float32 if f32 else torch.bfloat16
        dx = None if only_dw else torch.empty((t, k), dtype=dt, device="cuda")
        dw = torch.empty((n_out, k), dtype=dt, device="cuda")
        sbl.backward(layer, _dev(x), _dev(dy), t, dx, dw, flags | (sbl.SBL_GRAD_F32 if f32 else 0), workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(ws.cpu().numpy().view(np.uint16).reshape(t, k), xhat_ref)
        if f32:
            _close(dw.cpu().numpy(), dw_ref)
        else:
            _close(bd.bf16_to_f64(dw), dw_ref, rtol=BF16_REL, atol=ATOL)
        if not only_dw:
            dx_plain = torch.empty_like(dx)
            dw_plain = torch.empty_like(dw)
            sbl.backward(layer, _dev(x), _dev(dy), t, dx_plain, dw_plain, sbl.SBL_GRAD_F32 if f32 else 0)
            torch.cuda.synchronize()
            assert torch.equal(dx, dx_plain)
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


@pytest.mark.parametrize("k", [64, 1088, 2560, 3136, 16448])
def test_dequant_act_row_lengths(k):
    """xhat for a register-resident row length and for the long-row kernel."""
    n_out, t = 8, 5
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 52)))
    x = synth.activations(t, k, 53)
    dy = synth.upstream_grad(t, n_out, 54)
    ws = torch.empty((sbl.backward_workspace_bytes(t, k, sbl.SBL_DW_QUANT_X),), dtype=torch.uint8, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.float32, device="cuda")
    sbl.backward(layer, _dev(x), _dev(dy), t, None, dw, sbl.SBL_DW_QUANT_X | sbl.SBL_NO_DX | sbl.SBL_GRAD_F32,
                 workspace=ws)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(ws.cpu().numpy().view(np.uint16).reshape(t, k), oracle.dequant_act(xq_ref, ap_ref))
    _close(dw.cpu().numpy(), oracle.grad_w_quant_x(dy, x))


def _tie_rows(k):
    """Rows whose quotients 127|x| / a' hit exact half-integers (ties go to the
    even code), a row under the 1e-5 clamp, a Gaussian row, ties next to the
    bf16 maximum, and two rows whose a' has another significand than 254/128,
    where the only tie is |x| = a'/2 (quotient 63.5, code 64)."""
    rng = np.random.default_rng(61)
    rows = np.zeros((7, k), dtype=np.float32)
    halves = np.arange(0, 127) + 0.5                     # 0.5 .. 126.5, all bf16-exact
    rows[0, :127] = halves * rng.choice([-1.0, 1.0], 127)
    rows[0, 127] = 127.0                                 # a' = 127: quotient = |x|
    odd = np.arange(1, 254, 2, dtype=np.float32)          # a' = 254: quotient = |x| / 2
    rows[1, :odd.size] = odd * rng.choice([-1.0, 1.0], odd.size)
    rows[1, odd.size] = -254.0
    rows[2] = rng.uniform(-9e-6, 9e-6, size=k)            # every |x| < 1e-5: a' is the clamp
    rows[3] = rng.normal(size=k)
    # a' = 254 * 2^120 near the bf16 maximum: 127 |x| overflows fp32 for 253
    # and 251 times 2^120, so by the fp32 definition their codes saturate at
    # +-127 (the exact quotients would be the ties 126.5 and 125.5)
    rows[4, :4] = [254.0 * 2.0 ** 120, 253.0 * 2.0 ** 120, -251.0 * 2.0 ** 120, 1.0]
    # a' = 3: ties at +-1.5, beside values one bf16 step either side of 1.5
    # and a uniform fill
    rows[5] = rng.uniform(-2.9, 2.9, size=k)
    rows[5, 0] = 3.0
    rows[5, 5:k:37] = 1.5
    rows[5, 9:k:41] = -1.5
    rows[5, 3], rows[5, 4] = 1.5078125, -1.4921875
    # a' = 0.875 (a Gaussian row scaled under it): ties at +-0.4375
    rows[6] = np.clip(rng.normal(scale=0.25, size=k), -0.87, 0.87)
    rows[6, 1] = -0.875
    rows[6, 2:k:29] = 0.4375
    rows[6, 7:k:31] = -0.4375
    bits = synth.bits(torch.from_numpy(rows).to(torch.bfloat16))
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("gemv,k", [(False, 512), (True, 512), (False, 4096)])
def test_act_quant_exact_ties_and_clamp(gemv, k):
    """The division-free quantiser against the oracle's IEEE division on exact
    ties and on the clamped scale, in the act-quant kernels (one warp per row
    at k = 512, one block per row at 4096) and in the GEMV."""
    n_out = 64
    x = _tie_rows(k)
    t = x.shape[0]
    flags = sbl.SBL_PACK_GEMV if gemv else 0
    layer = sbl.Layer.allocate(n_out, k, 2, 4, flags)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 62)))
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    # the tie rows really are ties, and they went to the even code
    assert np.array_equal(np.abs(xq_ref[0, :127].astype(int)), 2 * np.round(np.arange(127) / 2 + 0.25).astype(int))
    assert (np.abs(xq_ref[1, :127].astype(int)) % 2 == 0).all()
    assert list(xq_ref[4, :3]) == [127, 127, -127]
    xb = x.float().numpy()
    for r, half in ((5, 1.5), (6, 0.4375)):
        tied = np.abs(xb[r]) == half
        assert tied.sum() > 20
        assert (np.abs(xq_ref[r][tied].astype(int)) == 64).all()


def _bf16_grid_rows(k):
    """One row per bf16 a' of two binades (256 rows): a' itself, then every
    bf16 magnitude of the 11 binades at and below a''s (those above a' left
    out), alternating signs, zero-filled: every quotient 127 |x| / a' down to
    code 0, ties included (a' = 254/128 * 2^e and powers of two among them)."""
    rows = np.zeros((256, k), dtype=np.float32)
    for r in range(256):
        e, mant = r // 128, r % 128
        ap = (1.0 + mant / 128.0) * 2.0 ** (e - 1)
        ex = np.arange(e - 11, e)[:, None]
        xs = ((1.0 + np.arange(128)[None, :] / 128.0) * 2.0 ** (ex - 0.0)).ravel()
        xs = xs[xs <= ap][: k - 1]
        xs = xs * np.where(np.arange(xs.size) % 2 == 0, 1.0, -1.0)
        rows[r, 0] = ap if r % 3 else -ap
        rows[r, 1:1 + xs.size] = xs
    return torch.from_numpy(rows).to(torch.bfloat16)


@pytest.mark.parametrize("k", [1536, 4096])
def test_act_quant_bf16_grid_bit_exact(k):
    """The division-free codes against the oracle's IEEE division for every
    bf16 value below a' in 11 binades, for all 256 bf16 a' of two binades, in
    the warp-per-row kernel (k = 1536) and the block-per-row kernel (the same
    values in 4096-wide rows), and the dequantised values xhat of both."""
    n_out = 64
    x = _bf16_grid_rows(k)
    t = x.shape[0]
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 68)))
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    # the grid reaches the ties and the whole code range
    assert (np.abs(xq_ref) == 64).sum() > 256 and (np.abs(xq_ref) == 127).sum() >= 256
    # the dequantising form of the same kernels (the dW operand xhat)
    dy = synth.upstream_grad(t, n_out, 69)
    flags = sbl.SBL_DW_QUANT_X | sbl.SBL_NO_DX | sbl.SBL_GRAD_F32
    ws = torch.empty((sbl.backward_workspace_bytes(t, k, flags),), dtype=torch.uint8, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.float32, device="cuda")
    sbl.backward(layer, _dev(x), _dev(dy), t, None, dw, flags, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(ws.cpu().numpy().view(np.uint16)[: t * k].reshape(t, k), oracle.dequant_act(xq_ref, ap_ref))


def test_act_quant_more_rows_than_resident_warps():
    """More token rows than the warp-per-row kernel keeps resident, so warps
    loop over rows."""
    n_out, k, t = 8, 256, 10000
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 63)))
    x = synth.activations(t, k, 64)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))


@pytest.mark.parametrize("t", [4, 8, 16, 33])
def test_decode_dispatch_both_paths_bit_exact(t):
    """A layer with the decode pack at the decode sizes: up to 32 tokens take
    the decode kernel (quantising for itself up to 4), more the 2:4
    tensor-core GEMM; both give the oracle's bits."""
    n_out, k = 6912, 2560
    w = synth.master_weights(n_out, k, 81)
    x = synth.activations(t, k, 82)
    layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_PACK_GEMV)
    sbl.prepare_weights(layer, _dev(w))
    assert sbl.forward_uses_gemv(layer, t) == (t <= 32)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    c0 = sbl.launch_count()
    sbl.forward(layer, _dev(x), t, y, xq, ap, acc)
    launched = sbl.launch_count() - c0
    torch.cuda.synchronize()
    ref = oracle.forward(w, x, 2, 4)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), ref["xq"])
    assert launched == (1 if t <= 4 else 2)  # the decode kernel alone, or act-quant first
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


NM_PATTERNS = [(6, 8), (4, 8), (3, 8), (1, 8), (2, 8), (5, 8), (7, 8), (8, 8), (1, 4), (3, 4), (4, 4), (1, 2), (2, 2)]


def _decode_check(n_out, k, n, m, t, seed, with_codes=True, flags=sbl.SBL_PACK_GEMV):
    """Prepare with the decode pack (its bytes checked against the oracle's
    pack), run sbl_forward at t tokens through the decode kernel and compare
    the int32 accumulators and y bit for bit (and the codes and scales it
    hands back)."""
    w = synth.master_weights(n_out, k, seed)
    x = synth.activations(t, k, seed + 1)
    layer = sbl.Layer.allocate(n_out, k, n, m, flags)
    sbl.prepare_weights(layer, _dev(w))
    torch.cuda.synchronize()
    ref = _check_prepared(layer, w, n, m)
    assert sbl.forward_uses_gemv(layer, t)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    if with_codes:
        xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
        ap = torch.empty((t,), dtype=torch.float32, device="cuda")
        sbl.forward(layer, _dev(x), t, y, xq, ap, acc)
    else:
        ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
        sbl.forward(layer, _dev(x), t, y, acc_debug=acc, workspace=ws)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    xq_ref, ap_ref = oracle.act_quant(x)
    if with_codes:
        assert np.array_equal(xq.cpu().numpy(), xq_ref)
        assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    acc_ref = oracle.gemm_acc(xq_ref, ref["weff"])
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    y_ref = oracle.dequant(acc_ref, ap_ref, ref["g"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), y_ref.view(np.uint32))
    _close(y.cpu().numpy(), y_ref)
    return layer


@pytest.mark.parametrize("n,m", NM_PATTERNS)
@pytest.mark.parametrize("t", [1, 3, 8, 9, 16, 32])
def test_decode_compressed_index_patterns(n, m, t):
    """Every N:M pattern through the compressed-index decode pack, on a shape
    with a ragged last row tile (136 rows) and a half 128-k unit (k = 448)."""
    _decode_check(136, 448, n, m, t, seed=700 + 16 * n + m + t)


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (1, 4), (8, 8)])
@pytest.mark.parametrize("t", [1, 5, 32])
def test_decode_smallest_layer(n, m, t):
    """The smallest layer the library takes (8 rows, k = 64): half a row tile
    and half a k unit, every other lane's weights padding."""
    _decode_check(8, 64, n, m, t, seed=760 + 8 * n + m + t)


CODE6 = sbl.SBL_PACK_GEMV | sbl.SBL_PACK_GEMV_6BIT


@pytest.mark.parametrize("n_out,k", [(136, 448), (8, 64), (264, 320)])
@pytest.mark.parametrize("t", [1, 3, 4, 5, 8, 9, 16, 32])
def test_decode_6bit_code(n_out, k, t):
    """2:4 layers with the 6-bit group code: the pack matches the oracle's
    streams and the decode kernel's accumulators and y match bit for bit, on
    ragged row tiles and half k units."""
    _decode_check(n_out, k, 2, 4, t, seed=1200 + n_out + t, flags=CODE6)


@pytest.mark.parametrize("n_out,k,t", [(11200, 640, 4), (11200, 640, 20), (16, 16384, 1), (16, 10240, 9)])
def test_decode_6bit_code_many_tiles_and_long_rows(n_out, k, t):
    _decode_check(n_out, k, 2, 4, t, seed=1300 + t, with_codes=False, flags=CODE6)


def test_decode_6bit_code_under_the_mask_from_codes_ablation():
    _decode_check(264, 320, 2, 4, 3, seed=1310, flags=CODE6 | sbl.SBL_MASK_FROM_QUANT)


FUSED_CASES = [
    # n_out, k, n, m, t
    (264, 320, 2, 4, 300),     # two 240-token tiles, the second ragged
    (256, 256, 2, 4, 16),
    (8, 64, 2, 4, 5),
    (520, 192, 1, 4, 33),
    (136, 448, 6, 8, 77),
    (384, 512, 8, 8, 260),
    (200, 128, 1, 2, 50),
    (264, 3072, 2, 4, 481),    # the longest rows the launch quantises itself
    (512, 1024, 4, 8, 1000),   # dense tiles of 192 or 256 tokens
]


@pytest.mark.parametrize("n_out,k,n,m,t", FUSED_CASES)
def test_fused_act_quant_forward(n_out, k, n, m, t):
    """SBL_FUSE_ACT_QUANT: one launch quantises the activations and runs the
    GEMM; codes, scales, accumulators and y match the oracle bit for bit."""
    w = synth.master_weights(n_out, k, 1400 + n_out + t)
    x = synth.activations(t, k, 1401 + t)
    layer = sbl.Layer.allocate(n_out, k, n, m, sbl.SBL_FUSE_ACT_QUANT)
    sbl.prepare_weights(layer, _dev(w))
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    ws = torch.full((sbl.workspace_bytes(t, k),), 0x5A, dtype=torch.uint8, device="cuda")  # stale counters
    c0 = sbl.launch_count()
    sbl.forward(layer, _dev(x), t, y, xq, ap, acc, workspace=ws)
    launched = sbl.launch_count() - c0
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    assert launched == 1  # the GEMM launch alone
    ref = oracle.forward(w, x, n, m)
    assert np.array_equal(xq.cpu().numpy(), ref["xq"])
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))
    # the codes in the workspace path too, and again over the counters it left
    y2 = torch.empty_like(y)
    for _ in range(2):
        sbl.forward(layer, _dev(x), t, y2, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int32), y2.view(torch.int32))


@pytest.mark.parametrize("t,k", [(300, 2560), (33, 6912), (5, 64), (4096, 2560)])
def test_quantize_activations_alone_then_forward_from_codes(t, k):
    """sbl_quantize_activations gives the oracle's codes and scales; the
    forward from them gives sbl_forward's y; a NaN sets the caller's word."""
    x = synth.activations(t, k, 1480 + t)
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sbl.quantize_activations(_dev(x), t, k, xq, ap, status)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    assert int(status.item()) == 0
    n_out = 256
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 1481)))
    y1 = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    sbl.forward_quantized(layer, xq, ap, t, y1)
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, _dev(x), t, y2, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    x[t // 2, k - 1] = float("nan")
    sbl.quantize_activations(_dev(x), t, k, xq, ap, status)
    torch.cuda.synchronize()
    assert int(status.item()) & sbl.SBL_STATUS_NONFINITE_X


def test_fused_act_quant_falls_back_without_a_workspace_or_on_long_rows():
    """Without a workspace (explicit code buffers) or with rows longer than
    3072 the flag leaves the two-launch path in place; same bits."""
    for (n_out, k, t, use_ws) in ((256, 512, 40, False), (256, 3584, 40, True)):
        w = synth.master_weights(n_out, k, 1450 + k)
        x = synth.activations(t, k, 1451)
        layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_FUSE_ACT_QUANT)
        sbl.prepare_weights(layer, _dev(w))
        y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
        xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
        ap = torch.empty((t,), dtype=torch.float32, device="cuda")
        ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda") if use_ws else None
        c0 = sbl.launch_count()
        sbl.forward(layer, _dev(x), t, y, xq, ap, workspace=ws)
        assert sbl.launch_count() - c0 == 2
        torch.cuda.synchronize()
        ref = oracle.forward(w, x, 2, 4)
        assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))


@pytest.mark.parametrize("t", [3, 40, 300])
def test_fused_act_quant_with_the_decode_pack(t):
    """A layer with both SBL_FUSE_ACT_QUANT and SBL_PACK_GEMV: decode-sized
    calls take the decode kernel, larger ones the GEMM that quantises in its
    own launch; the same bits either way."""
    n_out, k = 264, 1024
    w = synth.master_weights(n_out, k, 1470)
    x = synth.activations(t, k, 1471 + t)
    layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_FUSE_ACT_QUANT | sbl.SBL_PACK_GEMV)
    sbl.prepare_weights(layer, _dev(w))
    assert sbl.forward_uses_gemv(layer, t) == (t <= 32)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, _dev(x), t, y, acc_debug=acc, workspace=ws)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    ref = oracle.forward(w, x, 2, 4)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))


def test_fused_act_quant_flags_nonfinite_activations():
    n_out, k, t = 256, 2560, 300
    layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_FUSE_ACT_QUANT)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 1460)))
    x = synth.activations(t, k, 1461)
    x[250, 7] = float("nan")
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, _dev(x), t, y, workspace=ws)
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_ERR_NONFINITE and bits & sbl.SBL_STATUS_NONFINITE_X


@pytest.mark.parametrize("t,k", [(1, 2560), (3, 2560), (9, 2560), (2, 6912)])
def test_decode_nonfinite_activations_raise_status(t, k):
    """A non-finite activation in a decode call, quantised in the decode
    kernel (t <= 4) or by the act-quant kernel first, sets the status bit;
    clearing it restores SBL_OK on the next clean call."""
    n_out = 64
    layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_PACK_GEMV)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 64)))
    assert sbl.forward_uses_gemv(layer, t)
    x = synth.activations(t, k, 65)
    x[t - 1, k // 3] = float("nan") if t % 2 else float("inf")
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, _dev(x), t, y, workspace=ws)
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_ERR_NONFINITE and bits & sbl.SBL_STATUS_NONFINITE_X
    sbl.clear_status(layer)
    sbl.forward(layer, _dev(synth.activations(t, k, 66)), t, y, workspace=ws)
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


def test_act_quant_long_rows_flag_nonfinite():
    """Rows of 6912 (one block per row, the integer absmax): an Inf, a NaN and
    a finite row; the codes of the finite rows match the oracle and the status
    word records the non-finite input."""
    n_out, k, t = 64, 6912, 4
    layer = sbl.Layer.allocate(n_out, k, 6, 8)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 67)))
    x = synth.activations(t, k, 68)
    x[1, 100] = float("inf")
    x[2, 6911] = float("nan")
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    sbl.forward(layer, _dev(x), t, y, xq, ap)
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_ERR_NONFINITE and bits & sbl.SBL_STATUS_NONFINITE_X
    xq_ref, ap_ref = oracle.act_quant(x[[0, 3]])
    assert np.array_equal(xq.cpu().numpy()[[0, 3]], xq_ref)
    assert np.array_equal(ap.cpu().numpy()[[0, 3]].view(np.uint32), ap_ref.view(np.uint32))


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (8, 8)])
@pytest.mark.parametrize("t", [4, 20])
def test_decode_blocks_of_several_tiles(n, m, t):
    """11200 rows: three 16-row tiles per block and five units per tile, so a
    warp's units straddle two tiles and their partial sums meet in shared
    memory."""
    _decode_check(11200, 640, n, m, t, seed=900 + n + t, with_codes=False)


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8)])
@pytest.mark.parametrize("k,t", [(16384, 1), (16384, 8), (10240, 9)])
def test_decode_long_rows(n, m, k, t):
    """One tile of long rows: 128 (or 80) units over eight warps, each warp
    loading its 16 (or 10) units in two batches; 9 token rows of k = 10240 is
    about the most the kernel's shared memory holds."""
    _decode_check(16, k, n, m, t, seed=950 + n + t)


def test_decode_declines_rows_beyond_its_shared_memory():
    """17 token rows of k = 16384 (278 KB of codes) do not fit the decode
    kernel's shared memory: the call takes the tensor-core GEMM and still
    gives the oracle's bits."""
    n_out, k, t = 256, 16384, 17
    w = synth.master_weights(n_out, k, 960)
    x = synth.activations(t, k, 961)
    layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_PACK_GEMV)
    sbl.prepare_weights(layer, _dev(w))
    assert not sbl.forward_uses_gemv(layer, t)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, _dev(x), t, y, acc_debug=acc, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.forward(w, x, 2, 4)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))


@pytest.mark.parametrize("tiny", [2.0 ** -40, 0.0, -(2.0 ** -35)])
def test_gamma_midpoint_decided_by_a_tiny_magnitude(tiny):
    """8192 masters whose in-window magnitudes average exactly to the fp32
    midpoint 1 + 2^-24: alone that ties to even (1.0), and one magnitude far
    below the window (2^-40 or 2^-35) must round it up to 1 + 2^-23.  A scale
    decided from the in-window sum without the tiny magnitudes would miss it."""
    n_out, k = 32, 256
    v = np.ones(n_out * k, dtype=np.float32)
    v[0], v[1], v[2] = 3.0, 2.0 ** -11, tiny  # 8189 ones + 3 + 2^-11 + tiny
    w = torch.from_numpy(v.reshape(n_out, k)).to(torch.bfloat16)
    expect = 1.0 + 2.0 ** -23 if tiny != 0.0 else 1.0
    assert float(oracle.absmean_gamma(w)) == expect
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(w))
    gamma, g = sbl.read_scale(layer)
    assert gamma == expect and g == expect
    _check_prepared(layer, w, 2, 4)
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


def test_dw_quant_x_operand_on_tie_clamp_and_huge_rows():
    """xhat for rows with exact ties, the 1e-5 clamp, a Gaussian row and a row
    whose a' is past 2^120 (fp64 path): bit-exact against the oracle."""
    n_out, k = 64, 512
    x = _tie_rows(k)
    rows = x.float().numpy().copy()
    rows[2, :] *= 1.0  # keep the clamp row
    rows[3, :4] = [3.0e38, -1.5e38, 2.0e36, 1.0]  # a' past 2^120
    x = torch.from_numpy(rows).to(torch.bfloat16)
    t = x.shape[0]
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(synth.master_weights(n_out, k, 66)))
    dy = synth.upstream_grad(t, n_out, 67)
    flags = sbl.SBL_DW_QUANT_X | sbl.SBL_NO_DX | sbl.SBL_GRAD_F32
    ws = torch.empty((sbl.backward_workspace_bytes(t, k, flags),), dtype=torch.uint8, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.float32, device="cuda")
    sbl.backward(layer, _dev(x), _dev(dy), t, None, dw, flags, workspace=ws)
    torch.cuda.synchronize()
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(ws.cpu().numpy().view(np.uint16).reshape(t, k), oracle.dequant_act(xq_ref, ap_ref))
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


def test_masked_grad_with_dequantised_operand():
    """Both backward flags at once: dW = (dY^T . xhat) * mask, dX unchanged."""
    n_out, k, t = 264, 320, 70
    w = synth.master_weights(n_out, k, 95)
    x = synth.activations(t, k, 96)
    dy = synth.upstream_grad(t, n_out, 97)
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(w))
    ref = oracle.prepare(w, 2, 4)
    xq_ref, ap_ref = oracle.act_quant(x)
    dw_ref = oracle.grad_w_masked(dy, oracle.dequant_act(xq_ref, ap_ref), ref["mask"], 4)
    flags = sbl.SBL_MASKED_GRAD | sbl.SBL_DW_QUANT_X | sbl.SBL_GRAD_F32
    ws = torch.empty((sbl.backward_workspace_bytes(t, k, flags),), dtype=torch.uint8, device="cuda")
    dx = torch.empty((t, k), dtype=torch.float32, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.float32, device="cuda")
    sbl.backward(layer, _dev(x), _dev(dy), t, dx, dw, flags, workspace=ws)
    torch.cuda.synchronize()
    _close(dw.cpu().numpy(), dw_ref)
    assert (dw.cpu().numpy()[dw_ref == 0] == 0).all()
    _close(dx.cpu().numpy(), oracle.grad_x(dy, ref["weff"], ref["g"]))
    assert sbl.read_status(layer)[0] == sbl.SBL_OK


@pytest.mark.parametrize("n,m,flags,t", [(2, 4, 0, 300), (6, 8, 0, 300), (2, 4, sbl.SBL_PACK_GEMV, 3),
                                          (2, 4, sbl.SBL_PACK_GEMV, 12)])
def test_forward_from_codes_matches_forward(n, m, flags, t):
    """sbl_forward_quantized on the codes and scales sbl_forward wrote for x
    gives the same bits, on the 2:4 GEMM, the dense int8 GEMM and the GEMV
    (fused-quantisation sizes included), and so does a second layer sharing x."""
    n_out, k = 392, 512
    x = synth.activations(t, k, 98)
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    for seed in (99, 100):  # two layers sharing the activations, like q and k
        w = synth.master_weights(n_out, k, seed)
        layer = sbl.Layer.allocate(n_out, k, n, m, flags)
        sbl.prepare_weights(layer, _dev(w))
        y0 = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
        y1 = torch.full((t, n_out), float("nan"), dtype=torch.float32, device="cuda")
        acc1 = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
        if seed == 99:
            sbl.forward(layer, _dev(x), t, y0, xq, ap)
        else:
            ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
            sbl.forward(layer, _dev(x), t, y0, workspace=ws)
        sbl.forward_quantized(layer, xq, ap, t, y1, acc1)
        torch.cuda.synchronize()
        assert torch.equal(y0.view(torch.int32), y1.view(torch.int32))
        ref = oracle.forward(w, x, n, m)
        assert np.array_equal(acc1.cpu().numpy(), ref["acc"])
        assert sbl.read_status(layer)[0] == sbl.SBL_OK


def _row_sharded_prepare(w, n, m, shards):
    """Row shards of w through the three steps (sum words, word-wise sum,
    prepare from the sum); returns the shards' layers."""
    n_out, k = w.shape
    rows = n_out // shards
    layers, words = [], []
    for s in range(shards):
        wd = _dev(w[s * rows:(s + 1) * rows].contiguous())
        layer = sbl.Layer.allocate(rows, k, n, m)
        out = torch.full((sbl.SBL_SUM_WORDS,), -1, dtype=torch.int64, device="cuda")
        sbl.weight_abs_sum(layer, wd, out)
        layers.append((layer, wd))
        words.append(out)
    total = torch.stack(words).sum(0)
    for layer, wd in layers:
        sbl.prepare_weights_from_sum(layer, wd, total, n_out * k)
    torch.cuda.synchronize()
    return [layer for layer, _ in layers]


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8)])
@pytest.mark.parametrize("shards", [1, 2, 3])
@pytest.mark.parametrize("case", ["gaussian", "huge_in_one_shard"])
def test_row_sharded_prepare_matches_whole_tensor(n, m, shards, case):
    """Every row shard holds the whole tensor's gamma, mask and codes."""
    n_out, k = 384, 512
    w = synth.master_weights(n_out, k, 120 + shards)
    if case == "huge_in_one_shard":
        w[n_out - 5, 7] = 96.0  # >= 2^6: the exact path, from the last shard's bins
        w[3, 9] = 2.0 ** -40    # a tiny magnitude in the first shard
    ref = oracle.prepare(w, n, m)
    rows = n_out // shards
    for s, layer in enumerate(_row_sharded_prepare(w, n, m, shards)):
        gamma, g = sbl.read_scale(layer)
        assert np.float32(gamma).view(np.uint32) == np.float32(ref["gamma"]).view(np.uint32)
        assert np.float32(g) == ref["g"]
        assert np.array_equal(bd.mask(layer), ref["mask"][s * rows:(s + 1) * rows])
        assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"][s * rows:(s + 1) * rows])
        assert sbl.read_status(layer)[0] == sbl.SBL_OK


def test_row_sharded_midpoint_decided_by_a_tiny_magnitude_in_another_shard():
    """The midpoint construction (in-window mean exactly 1 + 2^-24) split in
    two shards, the one tiny magnitude in the second: both shards must round
    gamma up to 1 + 2^-23, as the whole tensor does."""
    v = np.ones(32 * 256, dtype=np.float32)
    v[0], v[1] = 3.0, 2.0 ** -11
    v[16 * 256 + 5] = 2.0 ** -40  # in the second shard's rows
    w = torch.from_numpy(v.reshape(32, 256)).to(torch.bfloat16)
    assert float(oracle.absmean_gamma(w)) == 1.0 + 2.0 ** -23
    for layer in _row_sharded_prepare(w, 2, 4, 2):
        assert sbl.read_scale(layer) == (1.0 + 2.0 ** -23, 1.0 + 2.0 ** -23)


GROUPS = [
    # (n_out, k, n, flags) per matrix; every group shares m
    (4, [(264, 320, 2, sbl.SBL_PACK_GEMV), (520, 192, 1, 0), (64, 64, 3, sbl.SBL_MASK_FROM_QUANT),
         (2560, 2560, 2, 0), (8, 64, 2, 0)]),
    (8, [(136, 448, 6, sbl.SBL_PACK_GEMV), (392, 832, 3, 0), (384, 512, 8, 0), (128, 384, 4, sbl.SBL_PACK_GEMV)]),
    (4, [(2560, 2560, 2, 0)] * 4 + [(6912, 2560, 2, 0)] * 2 + [(2560, 6912, 2, 0)]),  # a transformer block's linears
]


@pytest.mark.parametrize("m,mats", GROUPS)
def test_grouped_prepare_matches_one_call_per_layer(m, mats):
    """sbl_prepare_weights_grouped: every matrix's sections equal those of its
    own sbl_prepare_weights call and the oracle's, bit for bit."""
    layers, solo, ws = [], [], []
    for i, (n_out, k, n, flags) in enumerate(mats):
        w = synth.master_weights(n_out, k, 300 + i)
        if i == 1:
            w[3, 5] = 96.0  # one matrix with a magnitude outside the fast window
        ws.append(_dev(w))
        layers.append(sbl.Layer.allocate(n_out, k, n, m, flags))
        solo.append(sbl.Layer.allocate(n_out, k, n, m, flags))
        sbl.prepare_weights(solo[-1], ws[-1])
    sbl.prepare_weights_grouped(layers, ws)
    torch.cuda.synchronize()
    for i, (n_out, k, n, flags) in enumerate(mats):
        L = layers[i].layout()
        assert sbl.read_status(layers[i])[0] == sbl.SBL_OK
        assert sbl.read_scale(layers[i]) == sbl.read_scale(solo[i])
        # every section the prepare writes, padding included (the gaps between
        # sections are never written)
        spans = [(L.mask, n_out * k // m), (L.weff_bf16, 2 * n_out * k), (L.sp_values, n_out * k // 2),
                 (L.sp_meta, L.sp_meta_bytes), (L.codes, n_out * k), (L.gemv, L.gemv_bytes)]
        for off, size in spans:
            if off:
                assert torch.equal(layers[i].blob[off:off + size], solo[i].blob[off:off + size]), (i, off)
        from_codes = bool(flags & sbl.SBL_MASK_FROM_QUANT)
        if n_out * k <= 400 * 1024 and not from_codes:
            _check_prepared(layers[i], ws[i].cpu(), n, m)
        else:
            ref = oracle.prepare(ws[i].cpu(), n, m, mask_from_codes=from_codes)
            assert np.array_equal(bd.mask(layers[i]), ref["mask"])
            assert np.array_equal(bd.weff_from_bf16(layers[i]), ref["weff"])


def test_row_sharded_helper_orders_the_exchange_on_a_side_stream(monkeypatch):
    """sbl.prepare_weights_row_sharded with an explicit side stream: the
    exchange of the sum words runs on torch's current stream, and the
    preparation on the side stream must wait for it.  The stand-in exchange
    adds the other shard's words after a long sleep on the current stream, so
    a preparation that read the words early would decide gamma from this
    shard alone."""
    n_out, k = 384, 512
    rows = n_out // 2
    w = synth.master_weights(n_out, k, 77)
    w[rows + 5, 3] = 96.0  # the other shard moves gamma well away from this shard's own
    ref = oracle.prepare(w, 2, 4)
    other = sbl.Layer.allocate(rows, k, 2, 4)
    other_words = torch.empty(sbl.SBL_SUM_WORDS, dtype=torch.int64, device="cuda")
    sbl.weight_abs_sum(other, _dev(w[rows:].contiguous()), other_words)
    torch.cuda.synchronize()

    def exchange(words, group=None):
        torch.cuda._sleep(50_000_000)
        words.add_(other_words)
        return words

    monkeypatch.setattr(sbl, "allreduce_sum_words", exchange)
    side = torch.cuda.Stream()
    layer = sbl.Layer.allocate(rows, k, 2, 4)
    sbl.prepare_weights_row_sharded(layer, _dev(w[:rows].contiguous()), n_out, stream=side)
    torch.cuda.synchronize()
    gamma, g = sbl.read_scale(layer)
    assert np.float32(gamma).view(np.uint32) == np.float32(ref["gamma"]).view(np.uint32)
    assert np.array_equal(bd.mask(layer), ref["mask"][:rows])
    assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"][:rows])


def test_row_sharded_helper_over_a_one_rank_nccl_group():
    """The helper end to end over a real NCCL process group of one rank, with
    an explicit side stream: the whole tensor's gamma, mask and codes."""
    import socket

    import torch.distributed as dist

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        n_out, k = 256, 512
        w = synth.master_weights(n_out, k, 78)
        ref = oracle.prepare(w, 6, 8)
        side = torch.cuda.Stream()
        layer = sbl.Layer.allocate(n_out, k, 6, 8)
        sbl.prepare_weights_row_sharded(layer, _dev(w), n_out, stream=side)
        torch.cuda.synchronize()
        gamma, g = sbl.read_scale(layer)
        assert np.float32(gamma).view(np.uint32) == np.float32(ref["gamma"]).view(np.uint32)
        assert np.array_equal(bd.mask(layer), ref["mask"])
        assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"])
        assert sbl.read_status(layer)[0] == sbl.SBL_OK
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("t", [17000, 16000])
def test_sparse_forward_many_token_tiles(t):
    """256 weight rows at token counts on either side of one round of 240-token
    pair tiles (71 and 67 tiles), with ragged last tiles: the oracle's bits,
    with and without the accumulator output."""
    n_out, k = 256, 128
    w = synth.master_weights(n_out, k, 131)
    x = synth.activations(t, k, 132)
    layer = sbl.Layer.allocate(n_out, k, 2, 4)
    sbl.prepare_weights(layer, _dev(w))
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, _dev(x), t, y, acc_debug=acc, workspace=ws)
    y2 = torch.empty_like(y)
    sbl.forward(layer, _dev(x), t, y2, workspace=ws)  # the launch without accumulator output
    torch.cuda.synchronize()
    ref = oracle.forward(w, x, 2, 4)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
