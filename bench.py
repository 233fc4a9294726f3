"""Sparse-BitLinear benchmark on B200.

One step = the whole hot path of one Sparse-BitLinear layer over one batch:
prepare the weights (exact absmean, N:M mask from the masters, ternarise and
pack), the forward pass (per-token int8 activation quantisation, 2:4-sparse
int8 tensor-core GEMM with the dequant epilogue) and the dual-STE backward
(dX through the masked ternary weights, dense dW to every master).

Workload: the prefill-shaped FFN up projection, T=4096 tokens, K=2560,
N_out=6912, 2:4, bf16 masters ~N(0, 0.02), activations and upstream
gradients ~N(0, 1), seeded synthetic data.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs an independent replica on its own GPU with its
own token batch (no collective on the data path); the time is the max over
ranks and `value` counts the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Sparse-BitLinear fwd+bwd TOPS & tokens/s at 1 B200; % of sparse-int8/HBM roofline"
UNIT = "tokens/s"
WORKLOAD = dict(name="prefill 2:4 Sparse-BitLinear fwd+STE bwd, FFN up projection", tokens=4096, k=2560,
                n_out=6912, n=2, m=4)
ROTATE = 3  # distinct input sets cycled through the steps (3 x 112 MB > 126 MB L2)
SUSTAINED_STEPS = 2000  # about 0.6 s of back-to-back steps: the power-capped regime

# Algorithmic work of one step at this workload: the minimum bytes each HBM-bound
# kernel must move and the multiply-adds of each GEMM, the roofline numerators.
def algorithmic(T, K, N):
    dense_ops = 2.0 * T * K * N                    # one GEMM, dense-equivalent multiply-adds x 2
    return {
        "fwd_gemm_ops": dense_ops,                 # int8 x ternary, half of them skipped by 2:4
        "bwd_flops_each": dense_ops,               # dX and dW, bf16 x bf16 -> fp32
        "step_ops": 3.0 * dense_ops,
        "prep_bytes": N * K * 2 + N * K // 2 + N * K // 8,   # read W; write 2:4 values + metadata
        "actq_bytes": T * K * 2 + T * K + T * 4,            # read X; write xq + scales
        "fwd_bytes": N * K // 2 + N * K // 8 + T * K + T * 4 + T * N * 4,  # read W_eff, xq; write fp32 Y
        "dx_bytes": T * N * 2 + N * K * 2 + T * K * 2,
        "dw_bytes": T * N * 2 + T * K * 2 + N * K * 2,
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_linear_layers_bitlinear_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec.get(kernel_key)
        if ent and ent.get("source_sha") == kernel_source_sha():
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, every 20 ms)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            try:
                bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        names = [v for k, v in self.REASONS.items() if self.reasons & k and k != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# Distributed plumbing (one process per GPU)
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def sum_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(value: float, world: int) -> float:
    """The slowest rank's value (NCCL needs a device tensor, gloo a host one)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank: int, rotation: int, tensor: int) -> int:
    """Seed of one input tensor: every rank draws its own batch (weak scaling)."""
    return 1000 * rank + 10 * rotation + tensor


def exchange_dw(dw, world: int) -> None:
    """The one exchange of data-parallel training: every rank's dW summed over
    the ranks (in place; NCCL over NVLink on the GPU, gloo on the host).  The
    masters are the same on every rank, so the summed gradient updates them
    alike; the optimizer step that would scale and apply it is not part of
    the operator."""
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(dw, op=dist.ReduceOp.SUM)


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample, extrapolated linearly in tokens)
# ---------------------------------------------------------------------------
def oracle_sample(wb, xb, dyb, n, m, tokens):
    """Seconds for (prepare + act-quant over the whole batch, fwd + dX + dW over `tokens` tokens)."""
    import oracle

    t0 = time.perf_counter()
    p = oracle.prepare(wb, n, m)
    xq, ap = oracle.act_quant(xb)
    t_fixed = time.perf_counter() - t0
    t1 = time.perf_counter()
    acc = oracle.gemm_acc(xq[:tokens], p["weff"])
    oracle.dequant(acc, ap[:tokens], p["g"])
    oracle.grad_x(dyb[:tokens], p["weff"], p["g"])
    oracle.grad_w(dyb[:tokens], xb[:tokens])
    return t_fixed, time.perf_counter() - t1


class OracleFit:
    """Token-sampled oracle step time.

    The token part is linear in tokens plus a token-independent share (the
    n_out x k fp64 dW buffer is allocated and zeroed whatever the sample), so
    it is fitted from two sample sizes: intercept + slope * tokens.  `tokens`
    is sized so one sample takes about `target_s`.
    """

    def __init__(self, wb, xb, dyb, T, n, m, target_s):
        self.args = (wb, xb, dyb, n, m)
        self.T = T
        lo = min(8, T)
        _, v_lo = oracle_sample(*self.args, lo)
        mid = min(64, T)
        f_mid, v_mid = oracle_sample(*self.args, mid)
        # size from the per-token cost at `mid` (intercept included): an upper
        # bound on the slope, so the sample stays within its target
        self.tokens = int(max(mid, min(T, (target_s - f_mid) / max(v_mid / mid, 1e-9))))
        self.lo, self.v_lo = lo, v_lo
        self.step_s = self.sample()

    def sample(self):
        """One timed sample; returns the extrapolated full-step seconds."""
        f, v = oracle_sample(*self.args, self.tokens)
        slope = (v - self.v_lo) / (self.tokens - self.lo) if self.tokens > self.lo else 0.0
        if slope <= 0.0:  # timing noise on a small sample: no intercept, plain per-token cost
            slope, intercept = v / self.tokens, 0.0
        else:
            intercept = max(0.0, v - slope * self.tokens)
        return f + intercept + self.T * slope

    def describe(self, step_s):
        return (f"prepare and act-quant over the full batch, then fwd + dX + dW for {self.tokens} of {self.T} "
                f"tokens; the token part fitted as intercept + slope x tokens from samples of {self.lo} and "
                f"{self.tokens} tokens and extrapolated to {self.T} ({step_s:.1f} s per full step)")


def cpu_baseline(T, K, N, n, m, target_s=12.0, target_1t_s=10.0):
    """The oracle on all host cores, and on one thread beside it."""
    import oracle
    from sparse_linear_layers_bitlinear_b200 import synth

    wb = synth.bits(synth.master_weights(N, K, 0))
    xb = synth.bits(synth.activations(T, K, 1))
    dyb = synth.bits(synth.upstream_grad(T, N, 2))
    cores = oracle.threads()
    fit = OracleFit(wb, xb, dyb, T, n, m, target_s)
    oracle.set_threads(1)
    try:
        fit_1t = OracleFit(wb, xb, dyb, T, n, m, target_1t_s)
    finally:
        oracle.set_threads(cores)
    return {"value": T / fit.step_s, "unit": UNIT, "cores": cores, "nproc": os.cpu_count(), "kind": "oracle",
            "sample": fit.describe(fit.step_s),
            "single_thread": {"value": T / fit_1t.step_s, "unit": UNIT, "cores": 1,
                              "sample": fit_1t.describe(fit_1t.step_s)}}


def workload_config(world: int) -> dict:
    """The `config` object of both arms' JSON lines."""
    return {"workload": WORKLOAD["name"], "tokens": WORKLOAD["tokens"], "k": WORKLOAD["k"], "n_out": WORKLOAD["n_out"],
            "n": WORKLOAD["n"], "m": WORKLOAD["m"],
            "parallelism": f"data parallel x{world}" + (" (dW all-reduce each step)" if world > 1 else ""),
            "l2": f"inputs rotate over {ROTATE} seeded sets (3 x 112 MB > 126 MB L2)"}


def run_reference(args):
    """The oracle as the reference arm, timed on the host cores."""
    import oracle
    from sparse_linear_layers_bitlinear_b200 import synth

    T, K, N, n, m = (WORKLOAD[k] for k in ("tokens", "k", "n_out", "n", "m"))
    wb = synth.bits(synth.master_weights(N, K, 0))
    xb = synth.bits(synth.activations(T, K, 1))
    dyb = synth.bits(synth.upstream_grad(T, N, 2))
    # size each step's token sample so the whole run stays within ~2 minutes
    per_step = max(0.5, 120.0 / max(1, args.steps + args.warmup + 2))
    fit = OracleFit(wb, xb, dyb, T, n, m, per_step)
    for _ in range(args.warmup):
        fit.sample()
    t_run = time.perf_counter()
    est = [fit.sample() for _ in range(args.steps)]
    sample_s = (time.perf_counter() - t_run) / max(1, args.steps)  # wall seconds of one timed sample
    step_s = statistics.mean(est)
    value = T / step_s
    sample = ("per step: " + fit.describe(step_s) + "; ms_per_step is that extrapolated full step, "
              "sample_s_per_step the measured seconds of the sample behind it")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i64/f64", "data": "synthetic",
        "config": workload_config(args.gpus),
        "extrapolated": True,
        "sample_s_per_step": sample_s,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ---------------------------------------------------------------------------
# Other workloads, reported beside the headline line
# ---------------------------------------------------------------------------
def bench_decode(dev, hbm_gbs, reps=10):
    """Decode-shaped forward: T in {1, 4, 16, 32}, K = 2560, N_out in {2560,
    6912}, on layers prepared with the decode pack: 2:4 (2-bit codes and
    metadata, 2 bits a weight, or the 6-bit group code, 1.5 bits a weight) and
    6:8 (the compressed-index pack, 2.5 bits a weight).  One replay of a CUDA graph makes one call per distinct weight
    blob, the blobs holding more than 2 x L2 of packed weights, so every call
    streams its weights from HBM; the per-call time is the replay time over
    the calls and includes each call's launch inside the graph.  `floor_us`
    is the same chain of empty library launches (programmatic dependent
    launch, as every call is launched): what a chain of dependent calls pays
    before any work.  `hbm_frac` is the call's bytes (weights, bf16 x, fp32 y)
    over the per-call time against the measured HBM copy rate."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    K = 2560
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def per_call_us(body, calls, s):
        with torch.cuda.stream(s):
            for i in range(min(3, calls)):
                body(i)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(calls):
                body(i)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        del g
        return e0.elapsed_time(e1) / (calls * reps) * 1e3

    out = []
    floors = {}
    g6 = sbl.SBL_PACK_GEMV | sbl.SBL_PACK_GEMV_6BIT
    for (n, m, flags) in ((2, 4, sbl.SBL_PACK_GEMV), (2, 4, g6), (6, 8, sbl.SBL_PACK_GEMV)):
        for N in (2560, 6912):
            wbytes = sbl.prepared_layout(N, K, n, m, flags).gemv_bytes
            nblob = max(16, int(2.2 * 126e6 / wbytes) + 1)
            layers = []
            for i in range(nblob):
                L = sbl.Layer.allocate(N, K, n, m, flags, device=dev)
                sbl.prepare_weights(L, synth.master_weights(N, K, 5000 + i, device=dev))
                layers.append(L)
            s = torch.cuda.Stream(dev)
            if nblob not in floors:
                floors[nblob] = per_call_us(lambda i: sbl.selftest_chain_floor(sms, stream=s), nblob, s)
            for T in (1, 4, 16, 32):
                x = synth.activations(T, K, 7, device=dev)
                y = torch.empty((T, N), dtype=torch.float32, device=dev)
                ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
                us = per_call_us(lambda i: sbl.forward(layers[i], x, T, y, workspace=ws, stream=s), nblob, s)
                dec = sbl.forward_uses_gemv(layers[0], T)
                # weight bytes of the path taken: the decode pack, or the GEMM's int8 operand
                wb = wbytes if dec else (N * K * 0.625 if (n, m) == (2, 4) else N * K)
                by = wb + 2 * T * K + 4 * T * N
                floor = floors[nblob]
                out.append({"pattern": f"{n}:{m}", "pack": "6-bit group code" if flags & sbl.SBL_PACK_GEMV_6BIT
                            else ("2-bit codes + metadata" if (n, m) == (2, 4) else "compressed index"),
                            "n_out": N, "k": K, "tokens": T,
                            "path": "decode kernel" if dec else "tensor-core GEMM",
                            "us_per_call": us, "floor_us": floor, "tokens_per_s": T / (us * 1e-6),
                            "bytes_per_call": by, "gbs": by / (us * 1e-6) / 1e9,
                            "hbm_frac": by / (us * 1e-6) / 1e9 / hbm_gbs,
                            "over_floor_and_stream_us": us - floor - by / (hbm_gbs * 1e3),
                            "calls_per_replay": nblob})
            del layers
            torch.cuda.empty_cache()
    return {"workload": "decode forward on layers with the decode pack (2:4 at 2 bits a weight or its 6-bit group "
                        "code at 1.5, 6:8 compressed index at 2.5), K=2560; each call takes the faster path for its "
                        "size (`path`)",
            "timing": "CUDA graph of one call per distinct weight blob (> 2 x L2 of packed weights), per-call "
                      "time incl. launch; floor = the same chain of empty PDL launches",
            "points": out}


MMA_KINDS = {0: "2:4 int8 forward stage (256 x 240 x 256 logical k, with its metadata copy)",
             1: "dense int8 forward stage (256 x 256 x 128)",
             2: "bf16 backward stage (256 x 256 x 64)"}


def bench_mma_ceiling(dev, peaks, stages=2048, reps=5):
    """The rate each GEMM stage's MMA instructions reach with resident
    operands (sbl_selftest_mma_rate): one launch over every CTA pair, CUDA
    events around it, median of `reps` after 3 warm-up launches.  Returns per
    kind the rate in dense-equivalent TOPS beside its nominal peak (4x / 2x /
    1x the measured bf16 figure for 2:4 int8 / dense int8 / bf16)."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl

    pairs = torch.cuda.get_device_properties(dev).multi_processor_count // 2
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ratio = {0: 4.0, 1: 2.0, 2: 1.0}
    out = {}
    for kind, what in MMA_KINDS.items():
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for _ in range(3):
            macs = sbl.selftest_mma_rate(kind, stages, pairs, status)
        for a, b in evs:
            a.record()
            sbl.selftest_mma_rate(kind, stages, pairs, status)
            b.record()
        torch.cuda.synchronize(dev)
        assert int(status.item()) == 0, ("mma rate self test timed out", kind)
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        tops = 2.0 * macs * stages * pairs / (ms * 1e-3) / 1e12
        nominal = ratio[kind] * peaks["bf16_tflops"]
        out[{0: "sparse_i8", 1: "dense_i8", 2: "bf16"}[kind]] = {
            "what": what, "tops": tops, "nominal_tops": nominal, "frac_of_nominal": tops / nominal,
            "launch_ms": ms, "pairs": pairs, "stages_per_pair": stages}
    return out


def bench_prefill68(dev, peaks, ceiling=None, steps=20):
    """The 6:8 FFN down projection: T=4096, K=6912, N_out=2560, prepare +
    forward (dense int8 over W_eff codes) + dual-STE backward per step."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    T, K, N = 4096, 6912, 2560
    sets = [(synth.master_weights(N, K, 20 + 10 * r, device=dev), synth.activations(T, K, 21 + 10 * r, device=dev),
             synth.upstream_grad(T, N, 22 + 10 * r, device=dev)) for r in range(ROTATE)]
    layer = sbl.Layer.allocate(N, K, 6, 8, device=dev)
    y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
    dx = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def step(i, rec=False):
        w, x, dy = sets[i % ROTATE]
        if rec:
            ev[0].record()
        sbl.prepare_weights(layer, w)
        if rec:
            ev[1].record()
        sbl.forward(layer, x, T, y, workspace=ws)
        if rec:
            ev[2].record()
        sbl.backward(layer, x, dy, T, dx, dw, 0)
        if rec:
            ev[3].record()

    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    ph = [0.0, 0.0, 0.0]
    for i in range(5):
        step(i, True)
        torch.cuda.synchronize(dev)
        for j in range(3):
            ph[j] += ev[j].elapsed_time(ev[j + 1]) / 5
    # the dense int8 GEMM alone, from the codes of set 0 (events around each call)
    xq = torch.empty((T, K), dtype=torch.int8, device=dev)
    ap = torch.empty((T,), dtype=torch.float32, device=dev)
    sbl.prepare_weights(layer, sets[0][0])
    sbl.forward(layer, sets[0][1], T, y, xq, ap)
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
    for a, b in gev:
        a.record()
        sbl.forward_quantized(layer, xq, ap, T, y)
        b.record()
    torch.cuda.synchronize(dev)
    gemm_ms = statistics.median(a.elapsed_time(b) for a, b in gev)
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_OK, (code, bits)
    dense_ops = 2.0 * T * K * N
    i8_dense = 2.0 * peaks["bf16_tflops"] * 1e12
    gemm_tops = dense_ops / (gemm_ms * 1e-3) / 1e12
    ceil = ceiling["dense_i8"]["tops"] if ceiling else None
    return {"workload": "prefill 6:8 Sparse-BitLinear fwd+STE bwd, FFN down projection", "tokens": T, "k": K,
            "n_out": N, "n": 6, "m": 8, "ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3),
            "phase_ms": {"prepare": ph[0], "forward": ph[1], "backward": ph[2]},
            "fwd_dense_int8_tops": dense_ops / (ph[1] * 1e-3) / 1e12,
            "fwd_frac_of_dense_int8_peak": dense_ops / (ph[1] * 1e-3) / i8_dense,
            "gemm_ms": gemm_ms, "gemm_tops": gemm_tops, "gemm_frac_of_dense_int8_peak": gemm_tops * 1e12 / i8_dense,
            "gemm_frac_of_measured_ceiling": gemm_tops / ceil if ceil else None,
            "bwd_tflops": 2 * dense_ops / (ph[2] * 1e-3) / 1e12}


def bench_nm_sweep(dev, peaks, steps=10):
    """The N:M patterns the pages discuss, from dense ternary (8:8) down to
    2:8, plus 2:4 and 1:4, on the FFN down projection (T=4096, K=6912,
    N_out=2560): prepare + forward + dual-STE backward per step, CUDA events
    around each phase.  2:4 runs the 2:4-sparse tensor-core GEMM, every other
    pattern the dense int8 one over its W_eff codes."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    T, K, N = 4096, 6912, 2560
    sets = [(synth.master_weights(N, K, 40 + 10 * r, device=dev), synth.activations(T, K, 41 + 10 * r, device=dev),
             synth.upstream_grad(T, N, 42 + 10 * r, device=dev)) for r in range(ROTATE)]
    y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
    dx = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    dense_ops = 2.0 * T * K * N
    out = []
    for (n, m) in [(8, 8), (6, 8), (4, 8), (3, 8), (2, 8), (2, 4), (1, 4)]:
        layer = sbl.Layer.allocate(N, K, n, m, device=dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ph = [0.0, 0.0, 0.0]
        for i in range(steps + 3):
            w, x, dy = sets[i % ROTATE]
            ev[0].record()
            sbl.prepare_weights(layer, w)
            ev[1].record()
            sbl.forward(layer, x, T, y, workspace=ws)
            ev[2].record()
            sbl.backward(layer, x, dy, T, dx, dw, 0)
            ev[3].record()
            torch.cuda.synchronize(dev)
            if i >= 3:
                for j in range(3):
                    ph[j] += ev[j].elapsed_time(ev[j + 1]) / steps
        code, bits = sbl.read_status(layer)
        assert code == sbl.SBL_OK, (code, bits)
        peak = (4.0 if (n, m) == (2, 4) else 2.0) * peaks["bf16_tflops"]
        out.append({"n": n, "m": m, "kept_fraction": n / m, "ms_per_step": sum(ph),
                    "phase_ms": {"prepare": ph[0], "forward": ph[1], "backward": ph[2]},
                    "fwd_dense_equiv_tops": dense_ops / (ph[1] * 1e-3) / 1e12,
                    "fwd_kept_tops": dense_ops * n / m / (ph[1] * 1e-3) / 1e12,
                    "fwd_frac_of_int8_peak": dense_ops / (ph[1] * 1e-3) / 1e12 / peak,
                    "int8_peak": "2:4 sparse" if (n, m) == (2, 4) else "dense"})
        del layer
    return {"workload": "N:M sweep, FFN down projection T=4096, K=6912, N_out=2560, fwd + STE bwd",
            "timing": f"CUDA events around each phase, mean of {steps} steps after 3", "points": out}


def bench_fused_act_quant(dev, steps=40, reps=4):
    """A/B of SBL_FUSE_ACT_QUANT on the prefill 2:4 step (T=4096, K=2560,
    N_out=6912): the same step (prepare, forward, backward) with the
    activations quantised by their own kernel or inside the GEMM launch,
    alternated `reps` times on the same inputs; medians of the per-step time
    and of the prepare + forward part."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    T, K, N = 4096, 2560, 6912
    sets = [(synth.master_weights(N, K, 40 + 10 * r, device=dev), synth.activations(T, K, 41 + 10 * r, device=dev),
             synth.upstream_grad(T, N, 42 + 10 * r, device=dev)) for r in range(ROTATE)]
    y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
    dx = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    arms = {"separate kernel": 0, "inside the GEMM launch": sbl.SBL_FUSE_ACT_QUANT}
    layers = {name: sbl.Layer.allocate(N, K, 2, 4, f, device=dev) for name, f in arms.items()}
    step_us = {name: [] for name in arms}
    fwd_us = {name: [] for name in arms}

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(steps):
            fn(i)
        b.record()
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / steps * 1e3

    for _ in range(reps):
        for name, L in layers.items():
            def prep_fwd(i, L=L):
                w, x, _ = sets[i % ROTATE]
                sbl.prepare_weights(L, w)
                sbl.forward(L, x, T, y, workspace=ws)

            def step(i, L=L):
                prep_fwd(i)
                sbl.backward(L, sets[i % ROTATE][1], sets[i % ROTATE][2], T, dx, dw, 0)

            for i in range(3):
                step(i)
            step_us[name].append(timed(step))
            fwd_us[name].append(timed(prep_fwd))
            code, bits = sbl.read_status(L)
            assert code == sbl.SBL_OK, (code, bits)
    return {"workload": "prefill 2:4 step, T=4096, K=2560, N_out=6912", "steps_per_rep": steps, "reps": reps,
            "arms": {name: {"step_us": statistics.median(step_us[name]), "prepare_forward_us":
                            statistics.median(fwd_us[name]), "step_us_each": step_us[name]} for name in arms}}


def bench_ablations(dev, steps=10):
    """The pages' ablations and the STE reading variant as flags, on the
    prefill 2:4 workload: the plain step, the mask from the ternary codes
    (SBL_MASK_FROM_QUANT), the blocked gradient of pruned weights
    (SBL_MASKED_GRAD), and dW against the dequantised activations
    (SBL_DW_QUANT_X, which adds one quantise-and-dequantise pass).  CUDA events
    around each phase."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    T, K, N, n, m = (WORKLOAD[k] for k in ("tokens", "k", "n_out", "n", "m"))
    sets = [(synth.master_weights(N, K, 60 + 10 * r, device=dev), synth.activations(T, K, 61 + 10 * r, device=dev),
             synth.upstream_grad(T, N, 62 + 10 * r, device=dev)) for r in range(ROTATE)]
    y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
    bws = torch.empty(sbl.backward_workspace_bytes(T, K, sbl.SBL_DW_QUANT_X), dtype=torch.uint8, device=dev)
    dx = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    out = []
    for name, lflags, bflags in [("plain", 0, 0), ("mask_from_codes", sbl.SBL_MASK_FROM_QUANT, 0),
                                 ("masked_grad", 0, sbl.SBL_MASKED_GRAD), ("dw_quant_x", 0, sbl.SBL_DW_QUANT_X)]:
        layer = sbl.Layer.allocate(N, K, n, m, lflags, device=dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ph = [0.0, 0.0, 0.0]
        for i in range(steps + 3):
            w, x, dy = sets[i % ROTATE]
            ev[0].record()
            sbl.prepare_weights(layer, w)
            ev[1].record()
            sbl.forward(layer, x, T, y, workspace=ws)
            ev[2].record()
            sbl.backward(layer, x, dy, T, dx, dw, bflags, workspace=bws if bflags else None)
            ev[3].record()
            torch.cuda.synchronize(dev)
            if i >= 3:
                for j in range(3):
                    ph[j] += ev[j].elapsed_time(ev[j + 1]) / steps
        code, bits = sbl.read_status(layer)
        assert code == sbl.SBL_OK, (code, bits)
        out.append({"variant": name, "layer_flags": lflags, "backward_flags": bflags, "ms_per_step": sum(ph),
                    "phase_ms": {"prepare": ph[0], "forward": ph[1], "backward": ph[2]}})
        del layer
    return {"workload": WORKLOAD["name"], "timing": f"CUDA events around each phase, mean of {steps} steps after 3",
            "points": out}


def bench_train_step(dev, peaks, n, m, layers=30, tokens=8192, steps=3):
    """One training step's linear layers: 30 x {q, k, v, o: 2560 x 2560;
    gate, up: 2560 -> 6912; down: 6912 -> 2560} at 8192 tokens.  Per step every
    linear re-prepares its weights (mask and codes from its masters) and runs
    its forward; then every backward runs, last layer first.  Each linear has
    its own masters and upstream gradient; q, k and v share their input
    activations, as do gate and up (as in a transformer block), and each such
    group quantises them once (sbl_forward, then sbl_forward_quantized).  The
    whole step is one CUDA graph."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    H, F, T = 2560, 6912, tokens
    shapes = [("q", H, H), ("k", H, H), ("v", H, H), ("o", H, H), ("gate", F, H), ("up", F, H), ("down", H, F)]
    lead = {"k": "q", "v": "q", "up": "gate"}  # linears that take the activations of another
    lin = []
    for l in range(layers):
        by_name = {}
        for j, (name, n_out, k) in enumerate(shapes):
            seed = 1000 * l + 10 * j
            d = dict(layer=sbl.Layer.allocate(n_out, k, n, m, device=dev),
                     w=synth.master_weights(n_out, k, seed, device=dev),
                     dy=synth.upstream_grad(T, n_out, seed + 2, device=dev), n_out=n_out, k=k, shared=name in lead)
            if name in lead:
                d["x"], d["xq"], d["ap"] = (by_name[lead[name]][key] for key in ("x", "xq", "ap"))
            else:
                d["x"] = synth.activations(T, k, seed + 1, device=dev)
                d["xq"] = torch.empty((T, k), dtype=torch.int8, device=dev)
                d["ap"] = torch.empty((T,), dtype=torch.float32, device=dev)
            by_name[name] = d
            lin.append(d)
    # outputs reuse one buffer per shape (their values are not read within the step)
    y = {n_out: torch.empty((T, n_out), dtype=torch.float32, device=dev) for n_out in (H, F)}
    dx = {k: torch.empty((T, k), dtype=torch.bfloat16, device=dev) for k in (H, F)}
    dw = {(o, k): torch.empty((o, k), dtype=torch.bfloat16, device=dev) for (_, o, k) in shapes}
    s = torch.cuda.Stream(dev)

    # Grouped prepares per transformer block: q, k, v, o; gate, up; down
    # (each group's masters fit L2, so the second read of every matrix hits).
    groups = []
    for l in range(layers):
        blk = lin[7 * l:7 * l + 7]
        groups += [blk[0:4], blk[4:6], blk[6:7]]

    def prepare_phase_single():
        for d in lin:
            sbl.prepare_weights(d["layer"], d["w"], stream=s)

    def prepare_phase():
        for grp in groups:
            sbl.prepare_weights_grouped([d["layer"] for d in grp], [d["w"] for d in grp], stream=s)

    def forward_phase():
        for d in lin:
            if d["shared"]:
                sbl.forward_quantized(d["layer"], d["xq"], d["ap"], T, y[d["n_out"]], stream=s)
            else:
                sbl.forward(d["layer"], d["x"], T, y[d["n_out"]], d["xq"], d["ap"], stream=s)

    def backward_phase():
        for d in reversed(lin):
            sbl.backward(d["layer"], d["x"], d["dy"], T, dx[d["k"]], dw[(d["n_out"], d["k"])], 0, stream=s)

    def step():
        for grp in groups:
            sbl.prepare_weights_grouped([d["layer"] for d in grp], [d["w"] for d in grp], stream=s)
            for d in grp:
                if d["shared"]:
                    sbl.forward_quantized(d["layer"], d["xq"], d["ap"], T, y[d["n_out"]], stream=s)
                else:
                    sbl.forward(d["layer"], d["x"], T, y[d["n_out"]], d["xq"], d["ap"], stream=s)
        backward_phase()

    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    g.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    del g
    # The phases on their own: one graph per phase (all prepares; all
    # act-quants and forwards; all backwards), replayed in step order.
    graphs = []
    for body in (prepare_phase, forward_phase, backward_phase, prepare_phase_single):
        gp = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gp, stream=s):
            body()
        graphs.append(gp)
    for gp in graphs:
        gp.replay()
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    phase = [0.0, 0.0, 0.0, 0.0]
    for _ in range(steps):
        with torch.cuda.stream(s):
            for i, gp in enumerate(graphs):
                ev[i].record(s)
                gp.replay()
            ev[4].record(s)
        torch.cuda.synchronize(dev)
        for i in range(4):
            phase[i] += ev[i].elapsed_time(ev[i + 1]) / steps
    del graphs
    for d in lin[:7]:
        code, bits = sbl.read_status(d["layer"])
        assert code == sbl.SBL_OK, (code, bits)
    # roofline of the step at the measured peaks
    hbm, bf16 = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops_sustained"] * 1e12
    i8 = (4.0 if (n, m) == (2, 4) else 2.0) * bf16
    bound = {"prepare": 0.0, "forward": 0.0, "backward": 0.0}
    for (name, n_out, k) in shapes:
        ops = 2.0 * T * n_out * k
        prep_b = n_out * k * 2 + n_out * k * (0.625 if (n, m) == (2, 4) else 1.0)
        fwd_b = (0 if name in lead else T * k * 2) + T * k + T * n_out * 4  # shared inputs are quantised once
        bound["prepare"] += layers * prep_b / hbm
        bound["forward"] += layers * max(ops / i8, fwd_b / hbm)
        bound["backward"] += layers * 2 * ops / bf16
    total = sum(bound.values())
    del lin
    torch.cuda.empty_cache()
    names = ("prepare", "forward", "backward")
    return {"workload": f"training step, {layers} layers x 7 linears, {n}:{m}", "tokens": T, "n": n, "m": m,
            "ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3), "roofline_ms": total * 1e3,
            "roofline_frac": total * 1e3 / ms, "peak_note": "sustained bf16 peak (seconds-long step)",
            "phase_ms": dict(zip(names, phase[:3])),
            "prepare_one_launch_per_matrix_ms": phase[3],
            "prepare_note": "the step prepares each transformer block's linears in three grouped launches "
                            "(q, k, v, o; gate, up; down); prepare_one_launch_per_matrix_ms is the same phase "
                            "with one launch per matrix",
            "phase_roofline_ms": {k: v * 1e3 for k, v in bound.items()},
            "phase_frac": {k: bound[k] * 1e3 / phase[i] for i, k in enumerate(names)},
            "timing": f"one CUDA graph per step, {steps} replays after one warm-up; phase_ms: one graph per phase "
                      f"(all 210 prepares in 90 grouped launches; all act-quants and forwards; all backwards), "
                      f"replayed in step order, events between them"}


# ---------------------------------------------------------------------------
# Small fixed cases for a profiler (ncu): a few launches of one kernel family
# ---------------------------------------------------------------------------
def profile_decode():
    """The decode kernel at K = 2560, N_out = 6912: the 2:4 decode packs (a
    byte or 6 bits a group) and the 6:8 one, t = 1, 4 and 16 (t = 16 runs the
    act-quant kernel first), two calls each."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    dev = torch.device("cuda", 0)
    K, N = 2560, 6912
    g6 = sbl.SBL_PACK_GEMV | sbl.SBL_PACK_GEMV_6BIT
    for (n, m, flags) in ((2, 4, sbl.SBL_PACK_GEMV), (2, 4, g6), (6, 8, sbl.SBL_PACK_GEMV)):
        L = sbl.Layer.allocate(N, K, n, m, flags, device=dev)
        sbl.prepare_weights(L, synth.master_weights(N, K, 5000, device=dev))
        for T in (1, 4, 16):
            x = synth.activations(T, K, 7, device=dev)
            y = torch.empty((T, N), dtype=torch.float32, device=dev)
            ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
            for _ in range(2):
                sbl.forward(L, x, T, y, workspace=ws)
        torch.cuda.synchronize()


def profile_prefill68():
    """The 6:8 FFN down projection forward (T = 4096, K = 6912, N_out = 2560):
    act-quant (rows of 6912) and the dense int8 pair GEMM, three times."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    dev = torch.device("cuda", 0)
    T, K, N = 4096, 6912, 2560
    L = sbl.Layer.allocate(N, K, 6, 8, device=dev)
    sbl.prepare_weights(L, synth.master_weights(N, K, 0, device=dev))
    x = synth.activations(T, K, 1, device=dev)
    y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
    for _ in range(3):
        sbl.forward(L, x, T, y, workspace=ws)
    torch.cuda.synchronize()


def profile_grouped_prepare():
    """One transformer block's seven linears (q, k, v, o 2560 x 2560; gate, up
    2560 -> 6912; down 6912 -> 2560), 2:4, prepared in the three grouped
    launches of the training step, twice."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    dev = torch.device("cuda", 0)
    H, F = 2560, 6912
    shapes = [(H, H)] * 4 + [(F, H)] * 2 + [(H, F)]
    layers = [sbl.Layer.allocate(o, k, 2, 4, device=dev) for (o, k) in shapes]
    ws = [synth.master_weights(o, k, 10 * j, device=dev) for j, (o, k) in enumerate(shapes)]
    for _ in range(2):
        for a, b in ((0, 4), (4, 6), (6, 7)):
            sbl.prepare_weights_grouped(layers[a:b], ws[a:b])
    torch.cuda.synchronize()


def profile_prefill24():
    """The prefill 2:4 step (T = 4096, K = 2560, N_out = 6912, the benchmark's
    seeds): prepare, forward (act-quant and 2:4 GEMM) and backward, three steps
    on one input set: twelve launches."""
    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    dev = torch.device("cuda", 0)
    T, K, N = WORKLOAD["tokens"], WORKLOAD["k"], WORKLOAD["n_out"]
    w = synth.master_weights(N, K, 0, device=dev)
    x = synth.activations(T, K, 1, device=dev)
    dy = synth.upstream_grad(T, N, 2, device=dev)
    L = sbl.Layer.allocate(N, K, 2, 4, device=dev)
    y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
    dx = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        sbl.prepare_weights(L, w)
        sbl.forward(L, x, T, y, workspace=ws)
        sbl.backward(L, x, dy, T, dx, dw, 0)
    torch.cuda.synchronize()


PROFILE_CASES = {"decode": profile_decode, "prefill68": profile_prefill68, "grouped_prepare": profile_grouped_prepare,
                 "prefill24": profile_prefill24}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-extras", action="store_true", help="skip the decode and 6:8 workloads")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="run a few launches of one workload for a profiler and exit (no JSON line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.profile_case:
        PROFILE_CASES[args.profile_case]()
        return

    world, rank, local = dist_setup()
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    import torch

    from sparse_linear_layers_bitlinear_b200 import sbl, synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    T, K, N, n, m = (WORKLOAD[k] for k in ("tokens", "k", "n_out", "n", "m"))
    A = algorithmic(T, K, N)
    peaks = load_peaks()

    # Inputs: ROTATE seeded sets; the masters are the same on every rank (data
    # parallel), the activations and upstream gradients are each rank's own batch.
    sets = []
    for r in range(ROTATE):
        sets.append((synth.master_weights(N, K, replica_seed(0, r, 0), device=dev),
                     synth.activations(T, K, replica_seed(rank, r, 1), device=dev),
                     synth.upstream_grad(T, N, replica_seed(rank, r, 2), device=dev)))
    layer = sbl.Layer.allocate(N, K, n, m, device=dev)
    y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws = torch.empty(sbl.workspace_bytes(T, K), dtype=torch.uint8, device=dev)
    dx = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None, bwd=None):
        w, x, dy = sets[i % ROTATE]
        if ev is not None:
            ev[0].record(stream)
        sbl.prepare_weights(layer, w)
        if ev is not None:
            ev[1].record(stream)
        sbl.forward(layer, x, T, y, workspace=ws)
        if ev is not None:
            ev[2].record(stream)
        if bwd is not None:
            bwd[0].record(stream)
        sbl.backward(layer, x, dy, T, dx, dw, 0)  # dX and dW in one launch
        if bwd is not None:
            bwd[1].record(stream)
        exchange_dw(dw, world)  # the data-parallel gradient exchange (none on one GPU)
        if ev is not None:
            ev[3].record(stream)

    BWD_EVERY = 5  # steps whose backward launch is bracketed by events

    def timed(steps, bwd_events):
        """Device ms for `steps` back-to-back steps, the library launches they made,
        and the mean device ms of the backward launch, timed by events around it
        in every BWD_EVERY-th step (an event before it stops that launch from
        starting under the forward GEMM, so the other steps go without)."""
        bwd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               if bwd_events and i % BWD_EVERY == 0 else None for i in range(steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as clk:
            n0 = sbl.launch_count()
            start.record(stream)
            for i in range(steps):
                step(i, bwd=bwd[i])
            end.record(stream)
            n1 = sbl.launch_count()
            torch.cuda.synchronize(dev)
        barrier(world)
        bwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in bwd if e is not None) if bwd_events else None
        return start.elapsed_time(end), n1 - n0, bwd_ms, clk

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_OK, (code, bits)

    # The 2:4 forward GEMM alone, before the timed region (a kernel timed by
    # itself, against the burst peak): the forward from codes
    # (sbl_forward_quantized) on the activation codes of set 0, L2-resident as
    # in a step, where the act-quant kernel writes them just before; events
    # around each call.
    xq_b = torch.empty((T, K), dtype=torch.int8, device=dev)
    ap_b = torch.empty((T,), dtype=torch.float32, device=dev)
    sbl.prepare_weights(layer, sets[0][0])
    sbl.forward(layer, sets[0][1], T, y, xq_b, ap_b)
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
    for e_a, e_b in gev:
        e_a.record(stream)
        sbl.forward_quantized(layer, xq_b, ap_b, T, y)
        e_b.record(stream)
    torch.cuda.synchronize(dev)
    gemm_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in gev), world)
    # The rates the GEMMs' MMA instructions reach with resident operands.
    ceiling = bench_mma_ceiling(dev, peaks)

    # Timed region: the steps back to back.  Events sit only around the
    # backward launch of every fifth step.
    ms_total, launches, bwd_live_ms, clocks = timed(args.steps, True)
    ms_step = max_over_ranks(ms_total / args.steps, world)
    bwd_live_ms = max_over_ranks(bwd_live_ms, world)
    launches = int(sum_over_ranks(launches, world))
    code, bits = sbl.read_status(layer)
    assert code == sbl.SBL_OK, (code, bits)

    # Phase breakdown from separate, untimed steps with events between phases.
    n_phase = max(3, min(args.steps, 20))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_phase)]
    for i in range(n_phase):
        step(i, evs[i])
    torch.cuda.synchronize(dev)
    phase_ms = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j in range(3)]


    # End to end through the C ABI from pinned host buffers: every step copies
    # its inputs in (H2D), runs the step and copies its outputs back (D2H), all
    # inside the timed region.  Three streams pipeline consecutive steps the
    # way a training loop would: the inputs of step i+1 travel while step i
    # computes and the outputs of step i-1 travel back; two device buffer sets
    # alternate, and events keep each set's copies and compute in order.
    w_h = [s[0].cpu().pin_memory() for s in sets]
    x_h = [s[1].cpu().pin_memory() for s in sets]
    dy_h = [s[2].cpu().pin_memory() for s in sets]
    outs_h = [(torch.empty((T, N), dtype=torch.float32).pin_memory(),
               torch.empty((T, K), dtype=torch.bfloat16).pin_memory(),
               torch.empty((N, K), dtype=torch.bfloat16).pin_memory()) for _ in range(2)]
    ins_d = [tuple(torch.empty_like(t) for t in sets[0]) for _ in range(2)]
    outs_d = [(y, dx, dw), (torch.empty_like(y), torch.empty_like(dx), torch.empty_like(dw))]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b, r = i % 2, i % ROTATE
        w_d, x_d, dy_d = ins_d[b]
        y_d, dx_d, dw_d = outs_d[b]
        s_in.wait_event(ev_comp[b])  # the step two back no longer reads this input set
        with torch.cuda.stream(s_in):
            w_d.copy_(w_h[r], non_blocking=True)
            x_d.copy_(x_h[r], non_blocking=True)
            dy_d.copy_(dy_h[r], non_blocking=True)
        ev_in[b].record(s_in)
        s_comp.wait_event(ev_in[b])
        s_comp.wait_event(ev_out[b])  # the outputs of the step two back have left this set
        sbl.prepare_weights(layer, w_d, stream=s_comp)
        sbl.forward(layer, x_d, T, y_d, workspace=ws, stream=s_comp)
        sbl.backward(layer, x_d, dy_d, T, dx_d, dw_d, 0, stream=s_comp)
        with torch.cuda.stream(s_comp):
            exchange_dw(dw_d, world)  # ordered after the backward on the compute stream
        ev_comp[b].record(s_comp)
        s_out.wait_event(ev_comp[b])
        with torch.cuda.stream(s_out):
            for h_t, d_t in zip(outs_h[b], outs_d[b]):
                h_t.copy_(d_t, non_blocking=True)
        ev_out[b].record(s_out)

    def join_streams():
        for st in (s_in, s_comp, s_out):
            stream.wait_stream(st)

    for i in range(3):
        e2e_step(i)
    join_streams()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for st in (s_in, s_comp, s_out):
        st.wait_stream(stream)  # nothing of the timed steps starts before e0
    for i in range(args.e2e_steps):
        e2e_step(i)
    join_streams()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world)
    h2d = sum(t.numel() * t.element_size() for t in sets[0])
    d2h = y.numel() * 4 + dx.numel() * 2 + dw.numel() * 2

    # Rooflines: each phase's bound at the measured peaks.
    hbm = peaks["hbm_gbs"] * 1e9
    bf16 = peaks["bf16_tflops"] * 1e12
    i8_sparse = 4.0 * bf16  # dense-equivalent int8 2:4 peak: bf16 x (int8 2x, sparsity 2x) nominal ratio
    bound_ms = {
        "prepare": A["prep_bytes"] / hbm * 1e3,
        "forward": max(A["fwd_gemm_ops"] / i8_sparse, (A["actq_bytes"] + A["fwd_bytes"]) / hbm) * 1e3,
        "backward": max(2 * A["bwd_flops_each"] / bf16, (A["dx_bytes"] + A["dw_bytes"]) / hbm) * 1e3,
    }
    names = ["prepare", "forward", "backward"]
    dom = max(range(3), key=lambda j: phase_ms[j])
    dom_name = names[dom]
    if dom_name == "backward":
        achieved = 2 * A["bwd_flops_each"] / (bwd_live_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "traffic": ncu_traffic("bf16_backward"),
                "kernel": "k_gemm_pair<CfgPairDualBf16> (dX and dW, one launch)",
                "launch_ms": bwd_live_ms,
                "timing": "CUDA events around the backward launch of every 5th step inside the timed region, mean",
                "peak_note": f"{peaks['source']} bf16 burst figure (kernel timed inside a short step loop)"}
    else:
        by = {"prepare": A["prep_bytes"], "forward": A["actq_bytes"] + A["fwd_bytes"]}[dom_name]
        achieved = by / (phase_ms[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": ncu_traffic(dom_name), "kernel": dom_name,
                "peak_note": f"{peaks['source']} HBM copy bandwidth"}

    tokens_per_s = world * T / (ms_step * 1e-3)
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8xternary->i32 fwd, bf16->f32 bwd", "data": "synthetic",
        "config": workload_config(world),
        "tops": A["step_ops"] * world / (ms_step * 1e-3) / 1e12,
        "phase_ms": dict(zip(names, phase_ms)),
        "phase_roofline_ms": bound_ms,
        "step_roofline_frac": sum(bound_ms.values()) / ms_step,
        "roofline": roof,
        "fwd_gemm_roofline": {
            "bound": "tensor", "achieved": A["fwd_gemm_ops"] / (gemm_ms * 1e-3) / 1e12, "peak": 4.0 * peaks["bf16_tflops"],
            "unit": "TOPS (int8, dense-equivalent)", "frac": A["fwd_gemm_ops"] / (gemm_ms * 1e-3) / 1e12
            / (4.0 * peaks["bf16_tflops"]), "traffic": ncu_traffic("fwd_gemm"), "launch_ms": gemm_ms,
            "kernel": "k_gemm_pair<CfgPairSparse> (2:4 forward GEMM)",
            "timing": "CUDA events around each of 20 sbl_forward_quantized calls, median",
            "peak_note": f"2:4-sparse int8 = 4 x the {peaks['source']} bf16 burst figure (nominal ratio)",
            "measured_ceiling_tops": ceiling["sparse_i8"]["tops"],
            "frac_of_measured_ceiling": A["fwd_gemm_ops"] / (gemm_ms * 1e-3) / 1e12 / ceiling["sparse_i8"]["tops"]},
        "mma_ceiling": ceiling,
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "peaks": peaks,
    }
    if not args.no_extras:
        # The same step, back to back for long enough that the board's power
        # cap sets the clocks; its backward against the sustained GEMM peak.
        s_total, s_launches, s_bwd_ms, s_clocks = timed(SUSTAINED_STEPS, True)
        s_step = max_over_ranks(s_total / SUSTAINED_STEPS, world)
        s_bwd_ms = max_over_ranks(s_bwd_ms, world)
        s_tf = 2 * A["bwd_flops_each"] / (s_bwd_ms * 1e-3) / 1e12
        line["sustained"] = {
            "steps": SUSTAINED_STEPS, "ms_per_step": s_step, "value": world * T / (s_step * 1e-3), "unit": UNIT,
            "backward_launch_ms": s_bwd_ms, "backward_tflops": s_tf,
            "backward_frac_of_sustained_peak": s_tf / peaks["bf16_tflops_sustained"]
            if peaks.get("bf16_tflops_sustained") else None,
            "clocks": s_clocks.summary()}
        line["decode_gemv"] = bench_decode(dev, peaks["hbm_gbs"])
        line["prefill_6of8"] = bench_prefill68(dev, peaks, ceiling)
        line["train_step"] = [bench_train_step(dev, peaks, 2, 4), bench_train_step(dev, peaks, 4, 8)]
        line["nm_sweep"] = bench_nm_sweep(dev, peaks)
        line["ablations"] = bench_ablations(dev)
        line["fused_act_quant_ab"] = bench_fused_act_quant(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(T, K, N, n, m)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
