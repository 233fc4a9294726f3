"""ctypes binding of libsbl.so (include/sbl.h).

Argument marshalling only: every step of the operator runs in the CUDA
kernels of libsbl.so.  torch provides device memory and the current stream.
If the library is missing the import fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsbl.so")

# sbl_status
SBL_OK = 0
SBL_ERR_INVALID_ARG = 1
SBL_ERR_UNSUPPORTED_NM = 2
SBL_ERR_SHAPE = 3
SBL_ERR_ALIGN = 4
SBL_ERR_CUDA = 5
SBL_ERR_NONFINITE = 6
SBL_ERR_TIMEOUT = 7
SBL_ERR_DEVICE = 8
SBL_ERR_SCRATCH = 9
STATUS_NAMES = {
    0: "SBL_OK", 1: "SBL_ERR_INVALID_ARG", 2: "SBL_ERR_UNSUPPORTED_NM", 3: "SBL_ERR_SHAPE",
    4: "SBL_ERR_ALIGN", 5: "SBL_ERR_CUDA", 6: "SBL_ERR_NONFINITE", 7: "SBL_ERR_TIMEOUT", 8: "SBL_ERR_DEVICE",
    9: "SBL_ERR_SCRATCH",
}
# Fixed scratch of sbl_forward_noalloc (SBL_NOALLOC_SCRATCH_BYTES in include/sbl.h).
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
# layer flags
SBL_PACK_GEMV = 1 << 0
SBL_MASK_FROM_QUANT = 1 << 1
SBL_PACK_GEMV_6BIT = 1 << 2
SBL_FUSE_ACT_QUANT = 1 << 3
# backward flags
SBL_GRAD_F32 = 1 << 1
SBL_NO_DX = 1 << 2
SBL_NO_DW = 1 << 3
SBL_MASKED_GRAD = 1 << 4
SBL_DW_QUANT_X = 1 << 5
# device status bits
SBL_STATUS_NONFINITE_W = 1 << 0
SBL_STATUS_NONFINITE_X = 1 << 1
SBL_STATUS_TIMEOUT = 1 << 2


class SblError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


class sbl_layer(ctypes.Structure):
    _fields_ = [
        ("n_out", ctypes.c_int64),
        ("k", ctypes.c_int64),
        ("n", ctypes.c_int32),
        ("m", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("prepared", ctypes.c_void_p),
    ]


class sbl_blob_layout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_uint64) for name in (
        "total_bytes", "header", "mask", "codes", "weff_bf16", "sp_values", "sp_meta", "sp_meta_bytes",
        "gemv", "gamma", "g", "status", "scratch", "gemv_bytes")]


# Every entry point of include/sbl.h with its ctypes signature.
_P, _I64, _I32, _U32, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint64
_LP = ctypes.POINTER(sbl_layer)
SIGNATURES = {
    "sbl_prepared_layout": (_I32, [_I64, _I64, _I32, _I32, _U32, ctypes.POINTER(sbl_blob_layout)]),
    "sbl_prepared_bytes": (ctypes.c_size_t, [_I64, _I64, _I32, _I32, _U32]),
    "sbl_workspace_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "sbl_prepare_weights": (_I32, [_LP, _P, _P]),
    "sbl_prepare_weights_grouped": (_I32, [_LP, ctypes.POINTER(_P), _I32, _P]),
    "sbl_forward": (_I32, [_LP, _P, _I64, _P, _P, _P, _P, _P, _P]),
    "sbl_backward": (_I32, [_LP, _P, _P, _I64, _P, _P, _U32, _P]),
    "sbl_backward_ws": (_I32, [_LP, _P, _P, _I64, _P, _P, _U32, _P, _P]),
    "sbl_backward_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _U32]),
    "sbl_forward_noalloc": (_I32, [_LP, _P, _I64, _P, _P, _P]),
    "sbl_read_status": (_I32, [_LP, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "sbl_clear_status": (_I32, [_LP, _P]),
    "sbl_read_scale": (_I32, [_LP, _P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
    "sbl_selftest_wait_timeout": (_I32, [_P, _U64, _P]),
    "sbl_selftest_chain_floor": (_I32, [_I32, _P]),
    "sbl_quantize_activations": (_I32, [_P, _I64, _I64, _P, _P, _P, _P]),
    "sbl_selftest_mma_rate": (_I32, [_I32, _I32, _I32, _P, ctypes.POINTER(ctypes.c_int64), _P]),
    "sbl_version": (ctypes.c_char_p, []),
    "sbl_launch_count": (ctypes.c_uint64, []),
    "sbl_forward_uses_gemv": (ctypes.c_int, [_LP, _I64]),
    "sbl_weight_abs_sum": (_I32, [_LP, _P, _P, _P]),
    "sbl_prepare_weights_from_sum": (_I32, [_LP, _P, _P, _I64, _P]),
    "sbl_forward_quantized": (_I32, [_LP, _P, _P, _I64, _P, _P, _P]),
}

_lib = None


def lib():
    """Load libsbl.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_linear_layers_bitlinear_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(code: int, what: str):
    if code != SBL_OK:
        raise SblError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def prepared_layout(n_out: int, k: int, n: int, m: int, flags: int = 0) -> sbl_blob_layout:
    out = sbl_blob_layout()
    _check(lib().sbl_prepared_layout(n_out, k, n, m, flags, ctypes.byref(out)), "sbl_prepared_layout")
    return out


def prepared_bytes(n_out: int, k: int, n: int, m: int, flags: int = 0) -> int:
    return int(lib().sbl_prepared_bytes(n_out, k, n, m, flags))


def workspace_bytes(t: int, k: int) -> int:
    return int(lib().sbl_workspace_bytes(t, k))


@dataclass
class Layer:
    """A Sparse-BitLinear layer: shapes, N:M pattern and its prepared device blob."""

    n_out: int
    k: int
    n: int
    m: int
    flags: int
    blob: "object"  # torch.uint8 CUDA tensor

    @classmethod
    def allocate(cls, n_out: int, k: int, n: int, m: int, flags: int = 0, device="cuda"):
        import torch

        nbytes = prepared_bytes(n_out, k, n, m, flags)
        if nbytes == 0:
            prepared_layout(n_out, k, n, m, flags)  # raises with the reason
        blob = torch.empty(nbytes, dtype=torch.uint8, device=device)
        return cls(n_out, k, n, m, flags, blob)

    def c(self) -> sbl_layer:
        return sbl_layer(self.n_out, self.k, self.n, self.m, self.flags, self.blob.data_ptr())

    def layout(self) -> sbl_blob_layout:
        return prepared_layout(self.n_out, self.k, self.n, self.m, self.flags)

    def section(self, name: str, nbytes: int):
        off = getattr(self.layout(), name)
        return self.blob[off:off + nbytes]


def prepare_weights(layer: Layer, w_master, stream=None):
    cl = layer.c()
    _check(lib().sbl_prepare_weights(ctypes.byref(cl), _ptr(w_master), _stream(stream)), "sbl_prepare_weights")


def prepare_weights_grouped(layers, w_masters, stream=None):
    """sbl_prepare_weights_grouped: several layers (same m) prepared in one launch."""
    count = len(layers)
    arr = (sbl_layer * count)(*[L.c() for L in layers])
    ws = (_P * count)(*[_ptr(w) for w in w_masters])
    _check(lib().sbl_prepare_weights_grouped(arr, ws, count, _stream(stream)), "sbl_prepare_weights_grouped")


SBL_SUM_WORDS = 46


def weight_abs_sum(layer: Layer, w_shard, sum_out, stream=None):
    """sbl_weight_abs_sum: this shard's exact sum of |w| as SBL_SUM_WORDS words (int64 CUDA tensor)."""
    cl = layer.c()
    _check(lib().sbl_weight_abs_sum(ctypes.byref(cl), _ptr(w_shard), _ptr(sum_out), _stream(stream)),
           "sbl_weight_abs_sum")


def prepare_weights_from_sum(layer: Layer, w_shard, global_sum, global_numel: int, stream=None):
    """sbl_prepare_weights_from_sum: prepare this shard with the scale of the summed words."""
    cl = layer.c()
    _check(lib().sbl_prepare_weights_from_sum(ctypes.byref(cl), _ptr(w_shard), _ptr(global_sum), global_numel,
                                              _stream(stream)), "sbl_prepare_weights_from_sum")


def allreduce_sum_words(words, group=None):
    """Step 2 of the row-sharded scale: add every rank's sum words, word by
    word (an exact integer all-reduce; the words are below 2^63)."""
    import torch.distributed as dist

    dist.all_reduce(words, op=dist.ReduceOp.SUM, group=group)
    return words


def prepare_weights_row_sharded(layer: Layer, w_shard, global_rows: int, group=None, stream=None):
    """The three steps for this rank's row shard: its exact sum, the exact
    all-reduce of the words, and the preparation with the whole tensor's scale.

    The all-reduce is ordered on torch's current stream (as every collective
    is), so with an explicit ``stream`` the current stream first waits for the
    sum on ``stream``, and ``stream`` then waits for the all-reduce before the
    preparation reads the words.  No host synchronisation."""
    import torch

    words = torch.empty(SBL_SUM_WORDS, dtype=torch.int64, device=w_shard.device)
    weight_abs_sum(layer, w_shard, words, stream)
    cur = torch.cuda.current_stream(w_shard.device) if w_shard.is_cuda else None
    side = stream is not None and cur is not None and stream != cur
    if side:
        cur.wait_stream(stream)
    allreduce_sum_words(words, group)
    if side:
        stream.wait_stream(cur)
        words.record_stream(stream)
    prepare_weights_from_sum(layer, w_shard, words, global_rows * layer.k, stream)
    return words


def forward(layer: Layer, x, t: int, y, xq_out=None, xscale_out=None, acc_debug=None, workspace=None, stream=None):
    cl = layer.c()
    _check(lib().sbl_forward(ctypes.byref(cl), _ptr(x), t, _ptr(y), _ptr(xq_out), _ptr(xscale_out), _ptr(acc_debug),
                             _ptr(workspace), _stream(stream)), "sbl_forward")


def forward_quantized(layer: Layer, xq, xscale, t: int, y, acc_debug=None, stream=None):
    """sbl_forward_quantized: the forward from int8 codes and scales already at hand."""
    cl = layer.c()
    _check(lib().sbl_forward_quantized(ctypes.byref(cl), _ptr(xq), _ptr(xscale), t, _ptr(y), _ptr(acc_debug),
                                       _stream(stream)), "sbl_forward_quantized")


def quantize_activations(x, t: int, k: int, xq, xscale, status, stream=None):
    """sbl_quantize_activations: the forward's activation codes and scales
    alone; `status` is a device int32 tensor that receives the non-finite bit."""
    _check(lib().sbl_quantize_activations(_ptr(x), t, k, _ptr(xq), _ptr(xscale), _ptr(status), _stream(stream)),
           "sbl_quantize_activations")


def forward_noalloc(layer: Layer, x, t: int, y, acc_debug=None, stream=None):
    """sbl_forward_noalloc: the forward pass without any caller-provided scratch,
    for callers that cannot allocate device memory (see include/sbl.h)."""
    cl = layer.c()
    _check(lib().sbl_forward_noalloc(ctypes.byref(cl), _ptr(x), t, _ptr(y), _ptr(acc_debug), _stream(stream)),
           "sbl_forward_noalloc")


def backward(layer: Layer, x, dy, t: int, dx, dw, flags: int = 0, stream=None, workspace=None):
    """sbl_backward, or sbl_backward_ws when a workspace is given (SBL_DW_QUANT_X needs one)."""
    cl = layer.c()
    if workspace is None:
        _check(lib().sbl_backward(ctypes.byref(cl), _ptr(x), _ptr(dy), t, _ptr(dx), _ptr(dw), flags,
                                  _stream(stream)), "sbl_backward")
    else:
        _check(lib().sbl_backward_ws(ctypes.byref(cl), _ptr(x), _ptr(dy), t, _ptr(dx), _ptr(dw), flags,
                                     _ptr(workspace), _stream(stream)), "sbl_backward_ws")


def backward_workspace_bytes(t: int, k: int, flags: int) -> int:
    return int(lib().sbl_backward_workspace_bytes(t, k, flags))


def read_status(layer: Layer, stream=None):
    cl = layer.c()
    bits = ctypes.c_uint32(0)
    code = lib().sbl_read_status(ctypes.byref(cl), _stream(stream), ctypes.byref(bits))
    return code, int(bits.value)


def clear_status(layer: Layer, stream=None):
    cl = layer.c()
    _check(lib().sbl_clear_status(ctypes.byref(cl), _stream(stream)), "sbl_clear_status")


def read_scale(layer: Layer, stream=None):
    cl = layer.c()
    gamma, g = ctypes.c_float(0), ctypes.c_float(0)
    _check(lib().sbl_read_scale(ctypes.byref(cl), _stream(stream), ctypes.byref(gamma), ctypes.byref(g)),
           "sbl_read_scale")
    return gamma.value, g.value


def selftest_wait_timeout(status_dev, limit_ns: int, stream=None):
    _check(lib().sbl_selftest_wait_timeout(_ptr(status_dev), limit_ns, _stream(stream)), "sbl_selftest_wait_timeout")


def selftest_chain_floor(blocks: int, stream=None):
    """One empty kernel launched as the library launches its kernels (the
    per-call floor of a chain of dependent calls)."""
    _check(lib().sbl_selftest_chain_floor(blocks, _stream(stream)), "sbl_selftest_chain_floor")


def selftest_mma_rate(kind: int, stages: int, pairs: int, status, stream=None) -> int:
    """Resident-operand tensor-pipe rate launch of a GEMM stage (kind 0: 2:4
    int8 forward, 1: dense int8 forward, 2: bf16 backward); returns the
    multiply-adds of one pair's stage.  `status` is a device uint32 tensor."""
    macs = ctypes.c_int64(0)
    _check(lib().sbl_selftest_mma_rate(kind, stages, pairs, _ptr(status), ctypes.byref(macs), _stream(stream)),
           "sbl_selftest_mma_rate")
    return int(macs.value)


def version() -> str:
    return lib().sbl_version().decode()


def forward_uses_gemv(layer: Layer, t: int) -> bool:
    """Whether sbl_forward takes the decode kernel over the packed weights for t tokens on this layer."""
    cl = layer.c()
    return bool(lib().sbl_forward_uses_gemv(ctypes.byref(cl), t))


def launch_count() -> int:
    """Kernels the library has launched in this process (sbl_launch_count)."""
    return int(lib().sbl_launch_count())


class SparseBitLinear:
    """Convenience wrapper: one layer, its blob and its forward/backward buffers.

    All arithmetic happens in libsbl.so; this class only allocates torch
    tensors and calls the C ABI.
    """

    def __init__(self, n_out: int, k: int, n: int = 2, m: int = 4, flags: int = 0, device="cuda"):
        self.layer = Layer.allocate(n_out, k, n, m, flags, device)
        self.device = device

    def prepare(self, w_master):
        prepare_weights(self.layer, w_master)

    def forward(self, x, acc_debug: bool = False):
        import torch

        t = x.shape[0]
        y = torch.empty((t, self.layer.n_out), dtype=torch.float32, device=self.device)
        xq = torch.empty((t, self.layer.k), dtype=torch.int8, device=self.device)
        ap = torch.empty((max(t, 1),), dtype=torch.float32, device=self.device)
        acc = torch.empty((t, self.layer.n_out), dtype=torch.int32, device=self.device) if acc_debug else None
        forward(self.layer, x, t, y, xq, ap, acc)
        return y, xq, ap[:t], acc

    def backward(self, x, dy, f32: bool = False):
        import torch

        t = dy.shape[0]
        dt = torch.float32 if f32 else torch.bfloat16
        dx = torch.empty((t, self.layer.k), dtype=dt, device=self.device)
        dw = torch.empty((self.layer.n_out, self.layer.k), dtype=dt, device=self.device)
        backward(self.layer, x, dy, t, dx, dw, SBL_GRAD_F32 if f32 else 0)
        return dx, dw
