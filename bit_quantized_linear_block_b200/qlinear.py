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


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _bytes(n: int, device) -> torch.Tensor:
    """A zero-filled, 256-byte aligned device buffer (torch's caching
    allocator aligns to 512); workspaces must start zeroed."""
    return torch.zeros(max(int(n), 256), dtype=torch.uint8, device=device)


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
    assert W.dtype == torch.bfloat16 and W.is_cuda and W.dim() == 2 and W.is_contiguous()
    N, K = W.shape
    cfg = WeightCfg(fmt, int(bool(hadamard)) if fmt in (QL_W_NVFP4, QL_W_NVFP4_DECOMP) else 0, tau, alpha,
                    int(bool(expand_f16)), int(bool(expand_i8)), int(bool(keep_bf16)), 0)
    wbytes = lib.qlinear_weights_bytes(N, K, C.byref(cfg))
    wsbytes = lib.qlinear_prepare_ws_bytes(N, K, C.byref(cfg))
    if wbytes == 0:
        raise QLinearError("qlinear_weights_bytes", 2)
    buf = _bytes(wbytes, W.device)
    ws = _bytes(wsbytes, W.device)
    desc = Weights()
    _check("qlinear_prepare_weights",
           lib.qlinear_prepare_weights(_ptr(W), N, K, C.byref(cfg), _ptr(buf), buf.numel(),
                                       C.byref(desc), _ptr(ws), ws.numel(), _stream(stream)))
    pw = PackedWeights(desc, buf, N, K, fmt)
    pw._ws = ws      # keep the scratch alive until the stream has used it
    return pw


def qlinear_route(inp: torch.Tensor, out: torch.Tensor, threshold: float = 0.05, stream=None,
                  gamma: torch.Tensor | None = None, route: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None):
    """Returns device tensors (gamma float64 [1], route int32 [1]); reuses
    the given output and workspace tensors (a workspace stays valid across
    calls on one stream)."""
    assert inp.dtype == torch.bfloat16 and out.dtype == torch.bfloat16
    assert inp.shape == out.shape and inp.is_contiguous() and out.is_contiguous()
    n = inp.numel()
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float64, device=inp.device)
    if route is None:
        route = torch.empty(1, dtype=torch.int32, device=inp.device)
    if ws is None:
        ws = _bytes(lib.qlinear_route_ws_bytes(n), inp.device)
    _check("qlinear_route", lib.qlinear_route(_ptr(inp), _ptr(out), n, threshold, _ptr(gamma),
                                              _ptr(route), _ptr(ws), ws.numel(), _stream(stream)))
    return gamma, route


def qlinear_gamma_sums(inp: torch.Tensor, out: torch.Tensor, sums: torch.Tensor | None = None,
                       ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Device float64 [2]: (sum |out - in|, sum |in|) over these elements,
    this rank's share of Gamma when a block's tokens are split across ranks."""
    assert inp.dtype == torch.bfloat16 and out.dtype == torch.bfloat16
    assert inp.shape == out.shape and inp.is_contiguous() and out.is_contiguous()
    n = inp.numel()
    if sums is None:
        sums = torch.empty(2, dtype=torch.float64, device=inp.device)
    if ws is None:
        ws = _bytes(lib.qlinear_route_ws_bytes(n), inp.device)
    _check("qlinear_gamma_sums", lib.qlinear_gamma_sums(_ptr(inp), _ptr(out), n, _ptr(sums), _ptr(ws),
                                                        ws.numel(), _stream(stream)))
    return sums


def qlinear_route_from_sums(sums: torch.Tensor, threshold: float = 0.05, gamma: torch.Tensor | None = None,
                            route: torch.Tensor | None = None, stream=None):
    """Device tensors (gamma float64 [1], route int32 [1]) from the summed
    (sum |out - in|, sum |in|) of all ranks."""
    assert sums.dtype == torch.float64 and sums.is_cuda and sums.numel() == 2 and sums.is_contiguous()
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float64, device=sums.device)
    if route is None:
        route = torch.empty(1, dtype=torch.int32, device=sums.device)
    _check("qlinear_route_from_sums", lib.qlinear_route_from_sums(_ptr(sums), threshold, _ptr(gamma), _ptr(route),
                                                                  _stream(stream)))
    return gamma, route


def qlinear_tensor_amax(X: torch.Tensor, hadamard: bool = True, out: torch.Tensor | None = None,
                        ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Device fp32 [1]: max |H x| (or |x|) over the tensor."""
    assert X.dtype == torch.bfloat16 and X.is_cuda and X.dim() == 2 and X.is_contiguous()
    M, K = X.shape
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=X.device)
    if ws is None:
        ws = _bytes(lib.qlinear_quantize_ws_bytes(M, K, QL_ROUTE_NVFP4), X.device)
    _check("qlinear_tensor_amax", lib.qlinear_tensor_amax(_ptr(X), M, K, int(bool(hadamard)), _ptr(out),
                                                          _ptr(ws), ws.numel(), _stream(stream)))
    return out


def qlinear_quantize_act(X: torch.Tensor, act_fmt: int, hadamard: bool = True,
                         w: PackedWeights | None = None, rowmajor_scales: bool = True,
                         amax_in: torch.Tensor | None = None, out: dict | None = None, stream=None):
    """Quantized activations as a dict of device tensors (reuses `out`'s
    buffers when given)."""
    assert X.dtype == torch.bfloat16 and X.is_cuda and X.dim() == 2 and X.is_contiguous()
    M, K = X.shape
    dev = X.device
    if out is not None:
        _check("qlinear_quantize_act",
               lib.qlinear_quantize_act(_ptr(X), M, K, act_fmt, int(bool(hadamard)),
                                        C.byref(w.desc) if w is not None else None, _ptr(amax_in),
                                        _ptr(out["codes"]), _ptr(out["sf_mma"]), _ptr(out["sf_rowmajor"]),
                                        _ptr(out["scales"]), _ptr(out["_ws"]), out["_ws"].numel(),
                                        _stream(stream)))
        return out
    out = {}
    sf_mma = sf_rm = None
    if act_fmt in (QL_ROUTE_NVFP4, QL_ACT_NVFP4_DECOMP):
        kq = 2 * K if act_fmt == QL_ACT_NVFP4_DECOMP else K     # decomposed: [q1 | q2] per row
        codes = torch.empty((M, kq // 2), dtype=torch.uint8, device=dev)
        sf_mma = _bytes(lib.qlinear_sf_bytes(M, kq), dev)
        if rowmajor_scales:
            sf_rm = torch.empty((M, kq // 16), dtype=torch.uint8, device=dev)
        scales = torch.empty(1, dtype=torch.float32, device=dev)
    elif act_fmt in (QL_ROUTE_INT8, QL_ROUTE_INT6):
        codes = torch.empty((M, K), dtype=torch.int8, device=dev)
        scales = torch.empty(max(M, 1), dtype=torch.float32, device=dev)
    elif act_fmt in (QL_ACT_INT8_F16, QL_ACT_INT6_F16):
        codes = torch.empty((M, K), dtype=torch.float16, device=dev)
        scales = torch.empty(max(M, 1), dtype=torch.float32, device=dev)
    else:
        assert w is not None
        codes = torch.empty((M, w.desc.Kp), dtype=torch.int8, device=dev)
        scales = torch.empty(1, dtype=torch.float32, device=dev)
    ws = _bytes(lib.qlinear_quantize_ws_bytes(M, K, act_fmt), dev)
    wd = C.byref(w.desc) if w is not None else None
    _check("qlinear_quantize_act",
           lib.qlinear_quantize_act(_ptr(X), M, K, act_fmt, int(bool(hadamard)), wd, _ptr(amax_in),
                                    _ptr(codes), _ptr(sf_mma), _ptr(sf_rm), _ptr(scales), _ptr(ws),
                                    ws.numel(), _stream(stream)))
    out.update(codes=codes, sf_mma=sf_mma, sf_rowmajor=sf_rm, scales=scales, _ws=ws)
    return out


def qlinear_gemm(act_fmt: int, q: dict, M: int, w: PackedWeights, Y: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    dev = q["codes"].device
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=dev)
    _check("qlinear_gemm", lib.qlinear_gemm(act_fmt, _ptr(q["codes"]), _ptr(q.get("sf_mma")),
                                            _ptr(q["scales"]), M, C.byref(w.desc), _ptr(Y),
                                            _stream(stream)))
    return Y


class ForwardPlan:
    """Workspace for repeated qlinear_forward calls with fixed shapes."""

    def __init__(self, M: int, w: PackedWeights, route: int, device):
        self.M, self.w, self.route = M, w, route
        self.ws = _bytes(lib.qlinear_forward_ws_bytes(M, C.byref(w.desc), route), device)


def qlinear_forward(X: torch.Tensor, w: PackedWeights, route: int = QL_ROUTE_NVFP4,
                    Y: torch.Tensor | None = None, plan: ForwardPlan | None = None,
                    stream=None) -> torch.Tensor:
    assert X.dtype == torch.bfloat16 and X.is_cuda and X.dim() == 2 and X.is_contiguous()
    M, K = X.shape
    assert K == w.K
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    if plan is None:
        plan = ForwardPlan(M, w, route, X.device)
    _check("qlinear_forward",
           lib.qlinear_forward(_ptr(X), M, C.byref(w.desc), route, _ptr(Y), _ptr(plan.ws),
                               plan.ws.numel(), _stream(stream)))
    return Y


def qlinear_forward_routed(X: torch.Tensor, w: PackedWeights, route: torch.Tensor, Y: torch.Tensor | None = None,
                           ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Forward with the route read on the device (int32 [1] tensor, e.g. the
    router's output or a TDC state's next_route): no host synchronization."""
    assert X.dtype == torch.bfloat16 and X.is_cuda and X.dim() == 2 and X.is_contiguous()
    assert route.dtype == torch.int32 and route.is_cuda
    M, K = X.shape
    assert K == w.K
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = _bytes(lib.qlinear_forward_routed_ws_bytes(M, C.byref(w.desc)), X.device)
    _check("qlinear_forward_routed",
           lib.qlinear_forward_routed(_ptr(X), M, C.byref(w.desc), _ptr(route), _ptr(Y), _ptr(ws), ws.numel(),
                                      _stream(stream)))
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
    _check("qlinear_tdc_init", lib.qlinear_tdc_init(_ptr(cache.state_buf), _stream(stream)))


def qlinear_tdc_refresh(inp: torch.Tensor, out: torch.Tensor, cache: TdcCache, stream=None):
    """After computing the block: new delta, Gamma, E and the next decision (on the device)."""
    assert inp.dtype == torch.bfloat16 and out.dtype == torch.bfloat16 and inp.shape == out.shape
    assert inp.is_contiguous() and out.is_contiguous() and inp.numel() == cache.numel
    _check("qlinear_tdc_refresh",
           lib.qlinear_tdc_refresh(_ptr(inp), _ptr(out), cache.numel, _ptr(cache.slots[0]), _ptr(cache.slots[1]),
                                   _ptr(cache.state_buf), C.byref(cache.params), _ptr(cache.ws), cache.ws.numel(),
                                   _stream(stream)))


def qlinear_tdc_skip(inp: torch.Tensor, cache: TdcCache, out: torch.Tensor | None = None, stream=None):
    """Skip the block: out = bf16(in + latest delta)."""
    assert inp.dtype == torch.bfloat16 and inp.is_contiguous() and inp.numel() == cache.numel
    if out is None:
        out = torch.empty_like(inp)
    _check("qlinear_tdc_skip",
           lib.qlinear_tdc_skip(_ptr(inp), cache.numel, _ptr(cache.slots[0]), _ptr(cache.slots[1]),
                                _ptr(cache.state_buf), C.byref(cache.params), _ptr(out), _stream(stream)))
    return out


def qlinear_device_status(stream=None) -> int:
    v = C.c_int32(0)
    _check("qlinear_device_status", lib.qlinear_device_status(_stream(stream), C.byref(v)))
    return v.value


def qlinear_debug_set_wait_limit(cycles: int):
    lib.qlinear_debug_set_wait_limit(int(cycles))


def qlinear_debug_div_check(d: float, a_begin: int, count: int, stream=None) -> int:
    """Number of dividends (fp32 bit patterns a_begin .. a_begin+count-1)
    where the quantizer's block-scale division by d is not correctly rounded."""
    out = torch.zeros(1, dtype=torch.int64, device="cuda")
    _check("qlinear_debug_div_check", lib.qlinear_debug_div_check(float(d), int(a_begin), int(count),
                                                                  _ptr(out), _stream(stream)))
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
