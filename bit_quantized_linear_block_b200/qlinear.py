"""ctypes binding of libqlinear.so with torch tensors for device memory.

Each ``qlinear_*`` function here marshals torch tensors into the C entry
point of the same name (see ``include/qlinear.h``) and allocates outputs and
workspaces with torch.  No arithmetic of the method happens in Python: every
step runs in the library's CUDA kernels.  Importing this module loads the
library and fails loudly when it is missing.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlinear.so")

QL_OK = 0
STATUS_NAMES = {0: "QL_OK", 1: "QL_ERR_INVALID_ARG", 2: "QL_ERR_UNSUPPORTED_SHAPE",
                3: "QL_ERR_ALIGNMENT", 4: "QL_ERR_CUDA", 5: "QL_ERR_TIMEOUT",
                6: "QL_ERR_WORKSPACE", 7: "QL_ERR_NO_DEVICE"}
QL_W_NVFP4 = 0
QL_W_QARVD_INT4 = 2
QL_W_NVFP4_DECOMP = 3
QL_ROUTE_NVFP4 = 0
QL_ROUTE_INT8 = 1
QL_ACT_INT8_TENSOR = 2
QL_ACT_INT8_F16 = 3
QL_ACT_NVFP4_DECOMP = 4
QL_ROUTE_INT6 = 5
QL_ACT_INT6_F16 = 6
QL_ACT_INT6_TENSOR = 7
QL_ROUTE_BF16 = 8


class WeightCfg(C.Structure):
    _fields_ = [("fmt", C.c_int32), ("hadamard", C.c_int32), ("tau", C.c_float), ("alpha", C.c_float),
                ("expand_f16", C.c_int32), ("expand_i8", C.c_int32), ("keep_bf16", C.c_int32),
                ("reserved", C.c_int32)]


class Weights(C.Structure):
    _fields_ = [("fmt", C.c_int32), ("N", C.c_int32), ("K", C.c_int32), ("hadamard", C.c_int32),
                ("Kp", C.c_int32), ("reserved0", C.c_int32),
                ("codes", C.c_void_p), ("sf", C.c_void_p), ("gscale", C.c_void_p),
                ("outlier_mask", C.c_void_p), ("perm", C.c_void_p), ("gather", C.c_void_p),
                ("kinfo", C.c_void_p), ("s_norm", C.c_void_p), ("s_out", C.c_void_p),
                ("norms", C.c_void_p), ("w16", C.c_void_p), ("w8", C.c_void_p), ("wbf16", C.c_void_p)]


class TdcState(C.Structure):
    _fields_ = [("gamma", C.c_double), ("eps", C.c_double), ("acc", C.c_double), ("rho", C.c_double),
                ("n_delta", C.c_int32), ("cur", C.c_int32), ("skips", C.c_int32), ("last_skipped", C.c_int32),
                ("next_skip", C.c_int32), ("next_route", C.c_int32), ("steps", C.c_int32),
                ("reserved", C.c_int32)]


class TdcParams(C.Structure):
    _fields_ = [("gamma_threshold", C.c_float), ("eps_threshold", C.c_float), ("acc_max", C.c_float),
                ("max_skips", C.c_int32), ("kappa", C.c_float), ("rho_max", C.c_float)]


class QLinearError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -c 'import __graft_entry__ as g; g.build()'`")
    lib = C.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
    sig = {
        "qlinear_abi_version": (C.c_int, []),
        "qlinear_status_string": (C.c_char_p, [C.c_int]),
        "qlinear_device_status": (C.c_int, [vp, C.POINTER(i32)]),
        "qlinear_debug_set_wait_limit": (None, [C.c_longlong]),
        "qlinear_debug_div_check": (C.c_int, [f32, C.c_uint32, C.c_uint64, vp, vp]),
        "qlinear_sf_bytes": (sz, [i64, i32]),
        "qlinear_weights_bytes": (sz, [i32, i32, C.POINTER(WeightCfg)]),
        "qlinear_prepare_ws_bytes": (sz, [i32, i32, C.POINTER(WeightCfg)]),
        "qlinear_prepare_weights": (C.c_int, [vp, i32, i32, C.POINTER(WeightCfg), vp, sz,
                                              C.POINTER(Weights), vp, sz, vp]),
        "qlinear_route_ws_bytes": (sz, [i64]),
        "qlinear_route": (C.c_int, [vp, vp, i64, f32, vp, vp, vp, sz, vp]),
        "qlinear_gamma_sums": (C.c_int, [vp, vp, i64, vp, vp, sz, vp]),
        "qlinear_route_from_sums": (C.c_int, [vp, f32, vp, vp, vp]),
        "qlinear_quantize_ws_bytes": (sz, [i64, i32, i32]),
        "qlinear_tensor_amax": (C.c_int, [vp, i64, i32, i32, vp, vp, sz, vp]),
        "qlinear_quantize_act": (C.c_int, [vp, i64, i32, i32, i32, C.POINTER(Weights), vp, vp, vp,
                                           vp, vp, vp, sz, vp]),
        "qlinear_gemm": (C.c_int, [i32, vp, vp, vp, i64, C.POINTER(Weights), vp, vp]),
        "qlinear_forward_ws_bytes": (sz, [i64, C.POINTER(Weights), i32]),
        "qlinear_forward": (C.c_int, [vp, i64, C.POINTER(Weights), i32, vp, vp, sz, vp]),
        "qlinear_forward_routed_ws_bytes": (sz, [i64, C.POINTER(Weights)]),
        "qlinear_forward_routed": (C.c_int, [vp, i64, C.POINTER(Weights), vp, vp, vp, sz, vp]),
        "qlinear_tdc_init": (C.c_int, [vp, vp]),
        "qlinear_tdc_ws_bytes": (sz, [i64]),
        "qlinear_tdc_refresh": (C.c_int, [vp, vp, i64, vp, vp, vp, C.POINTER(TdcParams), vp, sz, vp]),
        "qlinear_tdc_skip": (C.c_int, [vp, i64, vp, vp, vp, C.POINTER(TdcParams), vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def _check(fn: str, status: int):
    if status != QL_OK:
        raise QLinearError(fn, status)


def _ptr(t: torch.Tensor | None):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream, device):
    """The stream handle to launch on: the given one (which must belong to
    `device`) or the current stream of `device`."""
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    if stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the call runs on {device}")
    return C.c_void_p(stream.cuda_stream)


def _tensor(t, name: str, dtype=None, device=None, min_bytes: int | None = None, dim: int | None = None):
    """Checks one tensor argument before anything reaches CUDA: a contiguous
    CUDA tensor, of `dtype` and on `device` when given, holding at least
    `min_bytes` bytes.  Raises TypeError or ValueError."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor, got one on {t.device}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call runs on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions, got {t.dim()}")
    if min_bytes is not None and t.numel() * t.element_size() < min_bytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, the call needs {min_bytes}")
    return t


def _weights(w) -> "PackedWeights":
    if not isinstance(w, PackedWeights):
        raise TypeError(f"w must be PackedWeights (from qlinear_prepare_weights), got {type(w).__name__}")
    return w


def _act_bytes(M: int, K: int, act_fmt: int, w=None) -> dict:
    """Bytes of each buffer of quantized activations [M, K] in `act_fmt`
    (K: the layer's input width; the Q-ARVD formats need their weights for
    the padded width Kp).  None: the format has no such buffer."""
    if act_fmt in (QL_ROUTE_NVFP4, QL_ACT_NVFP4_DECOMP):
        kq = 2 * K if act_fmt == QL_ACT_NVFP4_DECOMP else K      # decomposed: [q1 | q2] per row
        return dict(codes=M * kq // 2, sf_mma=lib.qlinear_sf_bytes(M, kq), sf_rowmajor=M * kq // 16, scales=4)
    if act_fmt in (QL_ROUTE_INT8, QL_ROUTE_INT6):
        return dict(codes=M * K, sf_mma=None, sf_rowmajor=None, scales=4 * max(M, 1))
    if act_fmt in (QL_ACT_INT8_F16, QL_ACT_INT6_F16):
        return dict(codes=2 * M * K, sf_mma=None, sf_rowmajor=None, scales=4 * max(M, 1))
    if act_fmt in (QL_ACT_INT8_TENSOR, QL_ACT_INT6_TENSOR):
        if w is None or w.fmt != QL_W_QARVD_INT4:
            raise ValueError("the per-tensor Q-ARVD formats need the Q-ARVD weights (w)")
        return dict(codes=M * w.desc.Kp, sf_mma=None, sf_rowmajor=None, scales=4)
    if act_fmt == QL_ROUTE_BF16:            # the unquantized bf16 input itself
        return dict(codes=2 * M * K, sf_mma=None, sf_rowmajor=None, scales=None)
    raise ValueError(f"unknown activation format {act_fmt}")


def _bytes(n: int, device) -> torch.Tensor:
    """A zero-filled, 256-byte aligned device buffer (torch's caching
    allocator aligns to 512); workspaces must start zeroed."""
    return torch.zeros(max(int(n), 256), dtype=torch.uint8, device=device)


_WEIGHT_SIZES = ("fmt", "N", "K", "hadamard", "Kp")
_WEIGHT_ARRAYS = ("codes", "sf", "gscale", "outlier_mask", "perm", "gather", "kinfo", "s_norm", "s_out", "norms",
                  "w16", "w8", "wbf16")


@dataclass
class PackedWeights:
    """Packed weights: the C descriptor plus the device buffer it points into."""
    desc: Weights
    buf: torch.Tensor
    N: int
    K: int
    fmt: int

    def view(self, field: str, dtype, count: int) -> torch.Tensor:
        """A tensor view of one of the descriptor's device arrays (inspection)."""
        addr = getattr(self.desc, field)
        off = addr - self.buf.data_ptr()
        itemsize = torch.empty(0, dtype=dtype).element_size()
        return self.buf[off:off + count * itemsize].view(dtype)

    def state_dict(self) -> dict:
        """Host copy for a checkpoint (torch.save): the descriptor's sizes,
        each array as a byte offset into the weight buffer (None for an
        absent one), and the buffer's bytes as a CPU uint8 tensor.  Copying
        the buffer waits for the work that wrote it."""
        base, end = self.buf.data_ptr(), self.buf.data_ptr() + self.buf.numel()
        offsets = {}
        for f in _WEIGHT_ARRAYS:
            p = getattr(self.desc, f)
            if p is None:
                offsets[f] = None
            elif base <= p < end:
                offsets[f] = p - base
            else:
                raise ValueError(f"weights array {f} does not point into the weight buffer")
        return {"abi": lib.qlinear_abi_version(),
                "sizes": {f: int(getattr(self.desc, f)) for f in _WEIGHT_SIZES},
                "offsets": offsets, "buf": self.buf.detach().to("cpu", copy=True)}

    @classmethod
    def from_state_dict(cls, sd: dict, device) -> "PackedWeights":
        """Packed weights on `device` from state_dict()'s output (same ABI
        version): the bytes are copied into a new buffer and every array
        pointer is rebased onto it."""
        if sd.get("abi") != lib.qlinear_abi_version():
            raise ValueError(f"packed weights of ABI {sd.get('abi')}, this library is ABI {lib.qlinear_abi_version()}")
        host = sd["buf"]
        if not isinstance(host, torch.Tensor) or host.dtype != torch.uint8 or host.dim() != 1:
            raise TypeError("state_dict['buf'] must be a 1-D uint8 tensor")
        buf = torch.empty(host.numel(), dtype=torch.uint8, device=device)
        buf.copy_(host)
        desc = Weights()
        for f in _WEIGHT_SIZES:
            setattr(desc, f, int(sd["sizes"][f]))
        for f in _WEIGHT_ARRAYS:
            off = sd["offsets"][f]
            if off is not None and not 0 <= off < buf.numel():
                raise ValueError(f"offset of {f} lies outside the weight buffer")
            setattr(desc, f, None if off is None else buf.data_ptr() + off)
        return cls(desc, buf, desc.N, desc.K, desc.fmt)


# ----------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ----------------------------------------------------------------------------

def qlinear_prepare_weights(W: torch.Tensor, fmt: int = QL_W_NVFP4, hadamard: bool = True,
                            tau: float = 3.5, alpha: float = 2.0, stream=None,
                            expand_f16: bool = False, expand_i8: bool = False,
                            keep_bf16: bool = False) -> PackedWeights:
    """expand_f16 (NVFP4 only) also keeps an f16 copy of the dequantized
    weights for the INT8 route's GEMM; expand_i8 (Q-ARVD only) keeps the
    INT4 codes sign-extended to int8 for the Q-ARVD GEMM; keep_bf16 (NVFP4
    only) keeps the bf16 weights for the unquantized QL_ROUTE_BF16 product."""
    _tensor(W, "W", torch.bfloat16, dim=2)
    dev = W.device
    N, K = W.shape
    cfg = WeightCfg(fmt, int(bool(hadamard)) if fmt in (QL_W_NVFP4, QL_W_NVFP4_DECOMP) else 0, tau, alpha,
                    int(bool(expand_f16)), int(bool(expand_i8)), int(bool(keep_bf16)), 0)
    wbytes = lib.qlinear_weights_bytes(N, K, C.byref(cfg))
    wsbytes = lib.qlinear_prepare_ws_bytes(N, K, C.byref(cfg))
    if wbytes == 0:
        raise QLinearError("qlinear_weights_bytes", 2)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        buf = _bytes(wbytes, dev)
        ws = _bytes(wsbytes, dev)
        desc = Weights()
        _check("qlinear_prepare_weights",
               lib.qlinear_prepare_weights(_ptr(W), N, K, C.byref(cfg), _ptr(buf), buf.numel(),
                                           C.byref(desc), _ptr(ws), ws.numel(), st))
    pw = PackedWeights(desc, buf, N, K, fmt)
    pw._ws = ws      # keep the scratch alive until the stream has used it
    return pw


def _block_pair(inp, out):
    _tensor(inp, "inp", torch.bfloat16)
    _tensor(out, "out", torch.bfloat16, inp.device)
    if inp.shape != out.shape:
        raise ValueError(f"inp {tuple(inp.shape)} and out {tuple(out.shape)} differ in shape")
    return inp.device, inp.numel()


def qlinear_route(inp: torch.Tensor, out: torch.Tensor, threshold: float = 0.05, stream=None,
                  gamma: torch.Tensor | None = None, route: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None):
    """Returns device tensors (gamma float64 [1], route int32 [1]); reuses
    the given output and workspace tensors (a workspace stays valid across
    calls on one stream)."""
    dev, n = _block_pair(inp, out)
    if gamma is not None:
        _tensor(gamma, "gamma", torch.float64, dev, 8)
    if route is not None:
        _tensor(route, "route", torch.int32, dev, 4)
    if ws is not None:
        _tensor(ws, "ws", torch.uint8, dev)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        if gamma is None:
            gamma = torch.empty(1, dtype=torch.float64, device=dev)
        if route is None:
            route = torch.empty(1, dtype=torch.int32, device=dev)
        if ws is None:
            ws = _bytes(lib.qlinear_route_ws_bytes(n), dev)
        _check("qlinear_route", lib.qlinear_route(_ptr(inp), _ptr(out), n, threshold, _ptr(gamma),
                                                  _ptr(route), _ptr(ws), ws.numel(), st))
    return gamma, route


def qlinear_gamma_sums(inp: torch.Tensor, out: torch.Tensor, sums: torch.Tensor | None = None,
                       ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Device float64 [2]: (sum |out - in|, sum |in|) over these elements,
    this rank's share of Gamma when a block's tokens are split across ranks."""
    dev, n = _block_pair(inp, out)
    if sums is not None:
        _tensor(sums, "sums", torch.float64, dev, 16)
    if ws is not None:
        _tensor(ws, "ws", torch.uint8, dev)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        if sums is None:
            sums = torch.empty(2, dtype=torch.float64, device=dev)
        if ws is None:
            ws = _bytes(lib.qlinear_route_ws_bytes(n), dev)
        _check("qlinear_gamma_sums", lib.qlinear_gamma_sums(_ptr(inp), _ptr(out), n, _ptr(sums), _ptr(ws),
                                                            ws.numel(), st))
    return sums


def qlinear_route_from_sums(sums: torch.Tensor, threshold: float = 0.05, gamma: torch.Tensor | None = None,
                            route: torch.Tensor | None = None, stream=None):
    """Device tensors (gamma float64 [1], route int32 [1]) from the summed
    (sum |out - in|, sum |in|) of all ranks."""
    _tensor(sums, "sums", torch.float64, min_bytes=16)
    dev = sums.device
    if gamma is not None:
        _tensor(gamma, "gamma", torch.float64, dev, 8)
    if route is not None:
        _tensor(route, "route", torch.int32, dev, 4)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        if gamma is None:
            gamma = torch.empty(1, dtype=torch.float64, device=dev)
        if route is None:
            route = torch.empty(1, dtype=torch.int32, device=dev)
        _check("qlinear_route_from_sums", lib.qlinear_route_from_sums(_ptr(sums), threshold, _ptr(gamma),
                                                                      _ptr(route), st))
    return gamma, route


def qlinear_tensor_amax(X: torch.Tensor, hadamard: bool = True, out: torch.Tensor | None = None,
                        ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Device fp32 [1]: max |H x| (or |x|) over the tensor."""
    _tensor(X, "X", torch.bfloat16, dim=2)
    dev = X.device
    M, K = X.shape
    if out is not None:
        _tensor(out, "out", torch.float32, dev, 4)
    if ws is not None:
        _tensor(ws, "ws", torch.uint8, dev)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty(1, dtype=torch.float32, device=dev)
        if ws is None:
            ws = _bytes(lib.qlinear_quantize_ws_bytes(M, K, QL_ROUTE_NVFP4), dev)
        _check("qlinear_tensor_amax", lib.qlinear_tensor_amax(_ptr(X), M, K, int(bool(hadamard)), _ptr(out),
                                                              _ptr(ws), ws.numel(), st))
    return out


_ACT_DTYPES = {QL_ROUTE_NVFP4: torch.uint8, QL_ACT_NVFP4_DECOMP: torch.uint8, QL_ROUTE_INT8: torch.int8,
               QL_ROUTE_INT6: torch.int8, QL_ACT_INT8_F16: torch.float16, QL_ACT_INT6_F16: torch.float16,
               QL_ACT_INT8_TENSOR: torch.int8, QL_ACT_INT6_TENSOR: torch.int8}


def qlinear_quantize_act(X: torch.Tensor, act_fmt: int, hadamard: bool = True,
                         w: PackedWeights | None = None, rowmajor_scales: bool = True,
                         amax_in: torch.Tensor | None = None, out: dict | None = None, stream=None):
    """Quantized activations as a dict of device tensors (reuses `out`'s
    buffers when given; they must be large enough for X)."""
    _tensor(X, "X", torch.bfloat16, dim=2)
    dev = X.device
    M, K = X.shape
    if w is not None:
        _weights(w)
    if act_fmt not in _ACT_DTYPES:
        raise ValueError(f"unknown activation format {act_fmt}")
    need = _act_bytes(M, K, act_fmt, w)
    if amax_in is not None:
        _tensor(amax_in, "amax_in", torch.float32, dev, 4)
    st = _stream(stream, dev)
    wd = C.byref(w.desc) if w is not None else None
    if out is not None:
        for key in ("codes", "sf_mma", "sf_rowmajor", "scales"):
            if out.get(key) is not None:
                _tensor(out[key], f"out[{key!r}]", None, dev, need[key] if need[key] is not None else 0)
        if need["sf_mma"] is not None and out.get("sf_mma") is None:
            raise ValueError("out['sf_mma'] is required for the NVFP4 formats")
        _tensor(out["_ws"], "out['_ws']", torch.uint8, dev)
        with torch.cuda.device(dev):
            _check("qlinear_quantize_act",
                   lib.qlinear_quantize_act(_ptr(X), M, K, act_fmt, int(bool(hadamard)), wd, _ptr(amax_in),
                                            _ptr(out["codes"]), _ptr(out.get("sf_mma")),
                                            _ptr(out.get("sf_rowmajor")), _ptr(out["scales"]), _ptr(out["_ws"]),
                                            out["_ws"].numel(), st))
        return out
    with torch.cuda.device(dev):
        if act_fmt in (QL_ROUTE_NVFP4, QL_ACT_NVFP4_DECOMP):
            kq = 2 * K if act_fmt == QL_ACT_NVFP4_DECOMP else K     # decomposed: [q1 | q2] per row
            codes = torch.empty((M, kq // 2), dtype=torch.uint8, device=dev)
            sf_mma = _bytes(need["sf_mma"], dev)
            sf_rm = torch.empty((M, kq // 16), dtype=torch.uint8, device=dev) if rowmajor_scales else None
        else:
            width = w.desc.Kp if act_fmt in (QL_ACT_INT8_TENSOR, QL_ACT_INT6_TENSOR) else K
            codes = torch.empty((M, width), dtype=_ACT_DTYPES[act_fmt], device=dev)
            sf_mma = sf_rm = None
        scales = torch.empty(need["scales"] // 4, dtype=torch.float32, device=dev)
        ws = _bytes(lib.qlinear_quantize_ws_bytes(M, K, act_fmt), dev)
        _check("qlinear_quantize_act",
               lib.qlinear_quantize_act(_ptr(X), M, K, act_fmt, int(bool(hadamard)), wd, _ptr(amax_in),
                                        _ptr(codes), _ptr(sf_mma), _ptr(sf_rm), _ptr(scales), _ptr(ws),
                                        ws.numel(), st))
    return dict(codes=codes, sf_mma=sf_mma, sf_rowmajor=sf_rm, scales=scales, _ws=ws)


def _output(Y, M: int, N: int, dev):
    if Y is None:
        return torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    return _tensor(Y, "Y", torch.bfloat16, dev, 2 * M * N)


def qlinear_gemm(act_fmt: int, q: dict, M: int, w: PackedWeights, Y: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """Y [M, N] bf16 from quantized activations `q` (qlinear_quantize_act's
    dict; for QL_ROUTE_BF16, {"codes": the bf16 input, "scales": None})."""
    _weights(w)
    M = int(M)
    if M < 0:
        raise ValueError(f"M must be >= 0, got {M}")
    need = _act_bytes(M, w.K, act_fmt, w if act_fmt in (QL_ACT_INT8_TENSOR, QL_ACT_INT6_TENSOR) else None)
    codes = _tensor(q["codes"], "q['codes']", None, None, need["codes"])
    dev = codes.device
    if need["sf_mma"] is not None and q.get("sf_mma") is not None:
        _tensor(q["sf_mma"], "q['sf_mma']", None, dev, need["sf_mma"])
    if need["scales"] is not None and q.get("scales") is not None:
        _tensor(q["scales"], "q['scales']", torch.float32, dev, need["scales"])
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        Y = _output(Y, M, w.N, dev)
        _check("qlinear_gemm", lib.qlinear_gemm(act_fmt, _ptr(codes), _ptr(q.get("sf_mma")), _ptr(q.get("scales")),
                                                M, C.byref(w.desc), _ptr(Y), st))
    return Y


class ForwardPlan:
    """Workspace for repeated qlinear_forward calls with fixed shapes."""

    def __init__(self, M: int, w: PackedWeights, route: int, device):
        self.M, self.w, self.route = M, _weights(w), route
        self.ws = _bytes(lib.qlinear_forward_ws_bytes(M, C.byref(w.desc), route), device)


def _layer_input(X, w):
    _tensor(X, "X", torch.bfloat16, dim=2)
    _weights(w)
    if X.shape[1] != w.K:
        raise ValueError(f"X has {X.shape[1]} columns, the weights take K = {w.K}")
    return X.device, X.shape[0]


def qlinear_forward(X: torch.Tensor, w: PackedWeights, route: int = QL_ROUTE_NVFP4,
                    Y: torch.Tensor | None = None, plan: ForwardPlan | None = None,
                    stream=None) -> torch.Tensor:
    dev, M = _layer_input(X, w)
    if plan is not None:
        _tensor(plan.ws, "plan.ws", torch.uint8, dev)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        Y = _output(Y, M, w.N, dev)
        if plan is None:
            plan = ForwardPlan(M, w, route, dev)
        _check("qlinear_forward",
               lib.qlinear_forward(_ptr(X), M, C.byref(w.desc), route, _ptr(Y), _ptr(plan.ws),
                                   plan.ws.numel(), st))
    return Y


def qlinear_forward_routed(X: torch.Tensor, w: PackedWeights, route: torch.Tensor, Y: torch.Tensor | None = None,
                           ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Forward with the route read on the device (int32 [1] tensor, e.g. the
    router's output or a TDC state's next_route): no host synchronization."""
    dev, M = _layer_input(X, w)
    _tensor(route, "route", torch.int32, dev, 4)
    if ws is not None:
        _tensor(ws, "ws", torch.uint8, dev)
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        Y = _output(Y, M, w.N, dev)
        if ws is None:
            ws = _bytes(lib.qlinear_forward_routed_ws_bytes(M, C.byref(w.desc)), dev)
        _check("qlinear_forward_routed",
               lib.qlinear_forward_routed(_ptr(X), M, C.byref(w.desc), _ptr(route), _ptr(Y), _ptr(ws), ws.numel(),
                                          st))
    return Y


# ----------------------------------------------------------------------------
# Temporal delta cache
# ----------------------------------------------------------------------------

class TdcCache:
    """Device buffers of one block's delta cache: two bf16 delta slots, the
    state (read with ``state()``) and the refresh workspace."""

    def __init__(self, numel: int, device, gamma_threshold=0.05, eps_threshold=0.1, acc_max=0.3,
                 max_skips=3, kappa=8.0, rho_max=1.0, stream=None):
        self.numel = int(numel)
        # each slot starts on a 16-byte boundary
        self.slots = torch.empty(2, max(8, (self.numel + 7) // 8 * 8), dtype=torch.bfloat16, device=device)
        self.state_buf = torch.zeros(C.sizeof(TdcState), dtype=torch.uint8, device=device)
        self.ws = _bytes(lib.qlinear_tdc_ws_bytes(self.numel), device)
        self.params = TdcParams(gamma_threshold, eps_threshold, acc_max, int(max_skips), kappa, rho_max)
        qlinear_tdc_init(self, stream)

    def state(self) -> TdcState:
        """Host copy of the device state (synchronizes with the device)."""
        return TdcState.from_buffer_copy(bytes(self.state_buf.cpu().numpy()))

    def delta(self, which: str = "latest") -> torch.Tensor:
        st = self.state()
        i = st.cur if which == "latest" else 1 - st.cur
        return self.slots[i, :self.numel]


def qlinear_tdc_init(cache: TdcCache, stream=None):
    dev = cache.state_buf.device
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check("qlinear_tdc_init", lib.qlinear_tdc_init(_ptr(cache.state_buf), st))


def _block_input(t, name, cache):
    _tensor(t, name, torch.bfloat16, cache.slots.device)
    if t.numel() != cache.numel:
        raise ValueError(f"{name} has {t.numel()} elements, the cache holds {cache.numel}")
    return t


def qlinear_tdc_refresh(inp: torch.Tensor, out: torch.Tensor, cache: TdcCache, stream=None):
    """After computing the block: new delta, Gamma, E and the next decision (on the device)."""
    _block_input(inp, "inp", cache)
    _block_input(out, "out", cache)
    dev = cache.slots.device
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check("qlinear_tdc_refresh",
               lib.qlinear_tdc_refresh(_ptr(inp), _ptr(out), cache.numel, _ptr(cache.slots[0]), _ptr(cache.slots[1]),
                                       _ptr(cache.state_buf), C.byref(cache.params), _ptr(cache.ws),
                                       cache.ws.numel(), st))


def qlinear_tdc_skip(inp: torch.Tensor, cache: TdcCache, out: torch.Tensor | None = None, stream=None):
    """Skip the block: out = bf16(in + latest delta)."""
    _block_input(inp, "inp", cache)
    if out is not None:
        _block_input(out, "out", cache)
    dev = cache.slots.device
    st = _stream(stream, dev)
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty_like(inp)
        _check("qlinear_tdc_skip",
               lib.qlinear_tdc_skip(_ptr(inp), cache.numel, _ptr(cache.slots[0]), _ptr(cache.slots[1]),
                                    _ptr(cache.state_buf), C.byref(cache.params), _ptr(out), st))
    return out


def qlinear_device_status(stream=None) -> int:
    """The current device's status word (0: no kernel has reported an error)."""
    v = C.c_int32(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    _check("qlinear_device_status", lib.qlinear_device_status(_stream(stream, dev), C.byref(v)))
    return v.value


def qlinear_debug_set_wait_limit(cycles: int):
    lib.qlinear_debug_set_wait_limit(int(cycles))


def qlinear_debug_div_check(d: float, a_begin: int, count: int, stream=None) -> int:
    """Number of dividends (fp32 bit patterns a_begin .. a_begin+count-1)
    where the quantizer's block-scale division by d is not correctly rounded."""
    dev = torch.device("cuda", torch.cuda.current_device())
    out = torch.zeros(1, dtype=torch.int64, device=dev)
    _check("qlinear_debug_div_check", lib.qlinear_debug_div_check(float(d), int(a_begin), int(count),
                                                                  _ptr(out), _stream(stream, dev)))
    return int(out.item())


# --- host-side layout helper for inspection (pure index permutation) --------

def sf_mma_to_rowmajor(sf_mma: torch.Tensor, rows: int, K: int) -> torch.Tensor:
    """Undo the MMA atom layout of block scales: returns uint8 [rows, K/16]."""
    kj = K // 16
    k_atoms = K // 64
    mpad = (rows + 127) // 128 * 128
    r = torch.arange(mpad, device=sf_mma.device)[:, None]
    j = torch.arange(kj, device=sf_mma.device)[None, :]
    off = ((r // 128) * k_atoms + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (j % 4)
    return sf_mma[: mpad * kj][off][:rows]
