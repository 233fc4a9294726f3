"""Full-size GPU parity at the benchmark workloads, through the same C ABI
calls the benchmark times.  Whole-array checks where the oracle is fast
(prepare outputs, activation codes), sampled outputs for the products."""
import numpy as np
import pytest
import torch

import oracle
from sparse_linear_layers_bitlinear_b200 import sbl, synth
from tests import blob_decode as bd

pytestmark = pytest.mark.gpu

WORKLOADS = [
    # name, n_out, k, n, m, t
    ("prefill 2:4, FFN up projection", 6912, 2560, 2, 4, 4096),
    ("prefill 6:8, FFN down projection", 2560, 6912, 6, 8, 4096),
]


def _samples(rng, rows, cols, count):
    r = rng.integers(0, rows, size=count)
    c = rng.integers(0, cols, size=count)
    edge_r = np.array([0, 127, 128, rows - 1, rows // 2] * 5)
    edge_c = np.array([0, 127, 128, 255, 256, cols - 1, cols // 2] * 5)[: len(edge_r)]
    return np.concatenate([r, edge_r]), np.concatenate([c, edge_c])


@pytest.mark.parametrize("name,n_out,k,n,m,t", WORKLOADS)
def test_fullsize_parity(name, n_out, k, n, m, t):
    w_d = synth.master_weights(n_out, k, 0, device="cuda")
    x_d = synth.activations(t, k, 1, device="cuda")
    dy_d = synth.upstream_grad(t, n_out, 2, device="cuda")
    w, x, dy = w_d.cpu(), x_d.cpu(), dy_d.cpu()

    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, w_d)
    torch.cuda.synchronize()
    ref = oracle.prepare(w, n, m)
    gamma, g, status = bd.header_scalars(layer)
    assert status == 0
    assert np.float32(gamma).view(np.uint32) == np.float32(ref["gamma"]).view(np.uint32)
    assert np.float32(g) == ref["g"]
    assert np.array_equal(bd.mask(layer), ref["mask"])
    assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"])
    if (n, m) == (2, 4):
        vals, meta = oracle.pack24(ref["weff"], ref["mask"])
        assert np.array_equal(bd.sp_values(layer), vals)
        assert np.array_equal(bd.sp_meta_canonical(layer)[0], meta)
    else:
        assert np.array_equal(bd.codes(layer), ref["weff"])

    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    sbl.forward(layer, x_d, t, y, xq, ap, acc)
    # the launch the benchmark times: workspace, no accumulator output
    y2 = torch.full((t, n_out), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, x_d, t, y2, workspace=ws)
    dx = torch.empty((t, k), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((n_out, k), dtype=torch.bfloat16, device="cuda")
    sbl.backward(layer, x_d, dy_d, t, dx, dw, 0)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))

    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))

    # Every accumulator and output: the oracle's codes times its W_eff in
    # float64 (a library matmul; the integer sums stay below 2^24, so fp64
    # holds them exactly), so every output tile of the GEMM's schedule is
    # checked, ragged last tiles included.
    acc_full = (xq_ref.astype(np.float64) @ ref["weff"].astype(np.float64).T)
    assert np.abs(acc_full).max() < 2 ** 31
    acc_full = acc_full.astype(np.int32)
    acc_h, y_h = acc.cpu().numpy(), y.cpu().numpy()
    assert np.array_equal(acc_h, acc_full)
    y_full = oracle.dequant(acc_full, ap_ref, ref["g"])
    assert np.array_equal(y_h.view(np.uint32), y_full.view(np.uint32))

    rng = np.random.default_rng(7)
    ti, oi = _samples(rng, t, n_out, 1500)
    accs = np.array([oracle.acc_at(xq_ref, ref["weff"], a, b) for a, b in zip(ti, oi)], dtype=np.int32)
    assert np.array_equal(acc_h[ti, oi], accs)
    y_ref = oracle.dequant(accs.reshape(-1, 1), ap_ref[ti], ref["g"]).ravel()
    assert np.array_equal(y_h[ti, oi].view(np.uint32), y_ref.view(np.uint32))

    dx_h = bd.bf16_to_f64(dx)
    ti, ki = _samples(rng, t, k, 600)
    dxr = np.array([oracle.grad_x_at(dy, ref["weff"], ref["g"], a, b) for a, b in zip(ti, ki)])
    err = np.abs(dx_h[ti, ki] - dxr)
    assert (err <= 1e-2 + 2.0 ** -7 * np.abs(dxr)).all(), err.max()

    dw_h = bd.bf16_to_f64(dw)
    oi, ki = _samples(rng, n_out, k, 600)
    dwr = np.array([oracle.grad_w_at(dy, x, a, b) for a, b in zip(oi, ki)])
    err = np.abs(dw_h[oi, ki] - dwr)
    assert (err <= 1e-2 + 2.0 ** -7 * np.abs(dwr)).all(), err.max()


@pytest.mark.parametrize("name,n_out,k,n,m,t", WORKLOADS)
@pytest.mark.parametrize("f32", [False, True])
def test_fullsize_gradients_whole_arrays(name, n_out, k, n, m, t, f32):
    """dX and dW of both prefill workloads, every element, in bf16 and in
    fp32 mode (SBL_GRAD_F32), against float64 products of the oracle's W_eff
    and scale (the oracle's gradient definitions, by a library matmul), plus
    sampled elements from the oracle itself."""
    w_d = synth.master_weights(n_out, k, 0, device="cuda")
    x_d = synth.activations(t, k, 1, device="cuda")
    dy_d = synth.upstream_grad(t, n_out, 2, device="cuda")
    layer = sbl.Layer.allocate(n_out, k, n, m)
    sbl.prepare_weights(layer, w_d)
    dt = torch.float32 if f32 else torch.bfloat16
    dx = torch.empty((t, k), dtype=dt, device="cuda")
    dw = torch.empty((n_out, k), dtype=dt, device="cuda")
    sbl.backward(layer, x_d, dy_d, t, dx, dw, sbl.SBL_GRAD_F32 if f32 else 0)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    ref = oracle.prepare(w_d.cpu(), n, m)
    dy64 = dy_d.cpu().double().numpy()
    x64 = x_d.cpu().double().numpy()
    dx_ref = (dy64 @ ref["weff"].astype(np.float64)) * np.float64(ref["g"])
    dw_ref = dy64.T @ x64
    rel = 1e-3 if f32 else 2.0 ** -7
    for got, want in ((dx, dx_ref), (dw, dw_ref)):
        g64 = got.double().cpu().numpy()
        err = np.abs(g64 - want)
        assert (err <= 1e-2 + rel * np.abs(want)).all(), err.max()
    rng = np.random.default_rng(17)
    ti, ki = _samples(rng, t, k, 200)
    dxr = np.array([oracle.grad_x_at(dy_d.cpu(), ref["weff"], ref["g"], a, b) for a, b in zip(ti, ki)])
    assert np.allclose(dx_ref[ti, ki], dxr, rtol=1e-12, atol=1e-12)
    oi, ki = _samples(rng, n_out, k, 200)
    dwr = np.array([oracle.grad_w_at(dy_d.cpu(), x_d.cpu(), a, b) for a, b in zip(oi, ki)])
    assert np.allclose(dw_ref[oi, ki], dwr, rtol=1e-12, atol=1e-12)


def test_fullsize_fused_act_quant_forward():
    """The prefill 2:4 workload (T = 4096, K = 2560, N_out = 6912) with the
    activations quantised inside the GEMM launch: every code, scale,
    accumulator and output."""
    n_out, k, t = 6912, 2560, 4096
    w_d = synth.master_weights(n_out, k, 0, device="cuda")
    x_d = synth.activations(t, k, 1, device="cuda")
    layer = sbl.Layer.allocate(n_out, k, 2, 4, sbl.SBL_FUSE_ACT_QUANT)
    sbl.prepare_weights(layer, w_d)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    xq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    ap = torch.empty((t,), dtype=torch.float32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, x_d, t, y, xq, ap, acc, workspace=ws)
    torch.cuda.synchronize()
    assert sbl.read_status(layer)[0] == sbl.SBL_OK
    ref = oracle.prepare(w_d.cpu(), 2, 4)
    xq_ref, ap_ref = oracle.act_quant(x_d.cpu())
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(ap.cpu().numpy().view(np.uint32), ap_ref.view(np.uint32))
    acc_full = (xq_ref.astype(np.float64) @ ref["weff"].astype(np.float64).T).astype(np.int32)
    assert np.array_equal(acc.cpu().numpy(), acc_full)
    y_ref = oracle.dequant(acc_full, ap_ref, ref["g"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), y_ref.view(np.uint32))


@pytest.mark.parametrize("t", [1, 4, 16, 32])
@pytest.mark.parametrize("n_out", [2560, 6912])
@pytest.mark.parametrize("n,m,flags", [(2, 4, sbl.SBL_PACK_GEMV), (6, 8, sbl.SBL_PACK_GEMV),
                                       (2, 4, sbl.SBL_PACK_GEMV | sbl.SBL_PACK_GEMV_6BIT)])
def test_decode_gemv_fullsize(t, n_out, n, m, flags):
    """The decode workload (k = 2560, n_out 2560 or 6912) through the decode
    kernel, 2:4 on its 2-bit pack or its 6-bit group code and 6:8 on the
    compressed-index pack: every accumulator and output, bit for bit."""
    k = 2560
    w_d = synth.master_weights(n_out, k, 10, device="cuda")
    x_d = synth.activations(t, k, 11, device="cuda")
    layer = sbl.Layer.allocate(n_out, k, n, m, flags)
    assert sbl.forward_uses_gemv(layer, t)
    sbl.prepare_weights(layer, w_d)
    y = torch.empty((t, n_out), dtype=torch.float32, device="cuda")
    acc = torch.empty((t, n_out), dtype=torch.int32, device="cuda")
    ws = torch.empty(sbl.workspace_bytes(t, k), dtype=torch.uint8, device="cuda")
    sbl.forward(layer, x_d, t, y, acc_debug=acc, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.forward(w_d.cpu(), x_d.cpu(), n, m)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))


@pytest.mark.parametrize("n,m", [(2, 4), (4, 8)])
@pytest.mark.parametrize("layer_index", [0, 29])
def test_fullsize_training_layer(n, m, layer_index):
    """One layer of the training-step workload at 8192 tokens: q, k, v, o
    (2560 x 2560), gate, up (2560 -> 6912), down (6912 -> 2560), with q/k/v and
    gate/up sharing their activations through sbl_forward_quantized as the
    benchmark runs them.  Prepare outputs whole, products sampled."""
    T, H, F = 8192, 2560, 6912
    shapes = [("q", H, H), ("k", H, H), ("v", H, H), ("o", H, H), ("gate", F, H), ("up", F, H), ("down", H, F)]
    lead = {"k": "q", "v": "q", "up": "gate"}
    rng = np.random.default_rng(11)
    acts = {}
    for j, (name, n_out, k) in enumerate(shapes):
        seed = 1000 * layer_index + 10 * j  # the benchmark's seeds for this layer
        w_d = synth.master_weights(n_out, k, seed, device="cuda")
        dy_d = synth.upstream_grad(T, n_out, seed + 2, device="cuda")
        layer = sbl.Layer.allocate(n_out, k, n, m)
        sbl.prepare_weights(layer, w_d)
        y = torch.empty((T, n_out), dtype=torch.float32, device="cuda")
        if name in lead:
            x_d, xq, ap, xq_ref, ap_ref = acts[lead[name]]
            sbl.forward_quantized(layer, xq, ap, T, y)
        else:
            x_d = synth.activations(T, k, seed + 1, device="cuda")
            xq = torch.empty((T, k), dtype=torch.int8, device="cuda")
            ap = torch.empty((T,), dtype=torch.float32, device="cuda")
            sbl.forward(layer, x_d, T, y, xq, ap)
            xq_ref, ap_ref = oracle.act_quant(x_d.cpu())
            acts[name] = (x_d, xq, ap, xq_ref, ap_ref)
        dx = torch.empty((T, k), dtype=torch.bfloat16, device="cuda")
        dw = torch.empty((n_out, k), dtype=torch.bfloat16, device="cuda")
        sbl.backward(layer, x_d, dy_d, T, dx, dw, 0)
        torch.cuda.synchronize()
        assert sbl.read_status(layer)[0] == sbl.SBL_OK, name

        w, x, dy = w_d.cpu(), x_d.cpu(), dy_d.cpu()
        ref = oracle.prepare(w, n, m)
        gamma, g, _ = bd.header_scalars(layer)
        assert np.float32(gamma).view(np.uint32) == np.float32(ref["gamma"]).view(np.uint32), name
        assert np.array_equal(bd.mask(layer), ref["mask"]), name
        assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"]), name
        if name not in lead:
            assert np.array_equal(xq.cpu().numpy(), xq_ref), name
        ti, oi = _samples(rng, T, n_out, 200)
        accs = np.array([oracle.acc_at(xq_ref, ref["weff"], a, b) for a, b in zip(ti, oi)], dtype=np.int32)
        y_ref = oracle.dequant(accs.reshape(-1, 1), ap_ref[ti], ref["g"]).ravel()
        assert np.array_equal(y.cpu().numpy()[ti, oi].view(np.uint32), y_ref.view(np.uint32)), name
        dx_h, dw_h = bd.bf16_to_f64(dx), bd.bf16_to_f64(dw)
        ti, ki = _samples(rng, T, k, 100)
        dxr = np.array([oracle.grad_x_at(dy, ref["weff"], ref["g"], a, b) for a, b in zip(ti, ki)])
        assert (np.abs(dx_h[ti, ki] - dxr) <= 1e-2 + 2.0 ** -7 * np.abs(dxr)).all(), name
        oi, ki = _samples(rng, n_out, k, 100)
        dwr = np.array([oracle.grad_w_at(dy, x, a, b) for a, b in zip(oi, ki)])
        assert (np.abs(dw_h[oi, ki] - dwr) <= 1e-2 + 2.0 ** -7 * np.abs(dwr)).all(), name


@pytest.mark.parametrize("n,m", [(2, 4), (4, 8)])
def test_training_step_prepares_all_210_matrices(n, m):
    """Every matrix of the 30-layer training step, drawn with the benchmark's
    seeds (layer l, projection j: seed 1000 l + 10 j): gamma, mask and W_eff
    of all 210 prepares, whole arrays."""
    H, F = 2560, 6912
    shapes = [(H, H), (H, H), (H, H), (H, H), (F, H), (F, H), (H, F)]
    layers = {(o, k): sbl.Layer.allocate(o, k, n, m) for (o, k) in set(shapes)}
    for l in range(30):
        for j, (n_out, k) in enumerate(shapes):
            w_d = synth.master_weights(n_out, k, 1000 * l + 10 * j, device="cuda")
            layer = layers[(n_out, k)]
            sbl.prepare_weights(layer, w_d)
            torch.cuda.synchronize()
            assert sbl.read_status(layer)[0] == sbl.SBL_OK
            ref = oracle.prepare(w_d.cpu(), n, m)
            gamma, _, _ = bd.header_scalars(layer)
            where = f"layer {l} projection {j}"
            assert np.float32(gamma).view(np.uint32) == np.float32(ref["gamma"]).view(np.uint32), where
            assert np.array_equal(bd.mask(layer), ref["mask"]), where
            assert np.array_equal(bd.weff_from_bf16(layer), ref["weff"]), where
