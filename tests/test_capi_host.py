"""Host-side checks of the C ABI that need no GPU: the library loads,
exports every entry point include/qlinear.h declares, and rejects bad
arguments before touching CUDA."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlinear.h")


@pytest.fixture(scope="module")
def ql():
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"QL_API\s+[\w\s\*]+?\b(qlinear_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for required in ("qlinear_prepare_weights", "qlinear_route", "qlinear_forward",
                     "qlinear_quantize_act", "qlinear_gemm", "qlinear_tensor_amax",
                     "qlinear_device_status", "qlinear_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(ql):
    out = subprocess.run(["nm", "-D", "--defined-only", ql.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(qlinear_\w+)", out))
    declared = set(declared_functions())
    assert declared, "no declarations parsed"
    assert declared <= exported, declared - exported
    for name in declared:
        getattr(ql.lib, name)              # resolvable through ctypes too


def test_abi_version_and_status_strings(ql):
    with open(HEADER) as f:
        ver = int(re.search(r"#define QLINEAR_ABI_VERSION (\d+)", f.read()).group(1))
    assert ql.lib.qlinear_abi_version() == ver
    assert ql.lib.qlinear_status_string(0) == b"ok"
    assert ql.lib.qlinear_status_string(5) == b"device wait timed out"
    assert ql.lib.qlinear_status_string(99) == b"unknown status"


def test_size_queries(ql):
    assert ql.lib.qlinear_sf_bytes(17776, 1920) == 17792 * 120      # rows padded to 128
    assert ql.lib.qlinear_sf_bytes(1, 128) == 128 * 8
    assert ql.lib.qlinear_sf_bytes(-1, 128) == 0 and ql.lib.qlinear_sf_bytes(4, 100) == 0
    cfg = ql.WeightCfg(ql.QL_W_NVFP4, 1, 3.5, 2.0)
    assert ql.lib.qlinear_weights_bytes(1920, 1920, C.byref(cfg)) >= 1920 * 960 + 1920 * 120
    assert ql.lib.qlinear_weights_bytes(1920, 1000, C.byref(cfg)) == 0          # K % 128
    ce = ql.WeightCfg(ql.QL_W_NVFP4, 1, 3.5, 2.0, 1, 0)                           # + f16 copy
    assert (ql.lib.qlinear_weights_bytes(1920, 1920, C.byref(ce))
            == ql.lib.qlinear_weights_bytes(1920, 1920, C.byref(cfg)) + 1920 * 1920 * 2)
    cq = ql.WeightCfg(ql.QL_W_QARVD_INT4, 0, 3.5, 2.0)
    assert ql.lib.qlinear_weights_bytes(384, 640, C.byref(cq)) >= 384 * (640 + 64) // 2
    cb = ql.WeightCfg(ql.QL_W_NVFP4, 1, 3.5, 2.0, 0, 0, 1)                        # + bf16 weights
    assert (ql.lib.qlinear_weights_bytes(1920, 1920, C.byref(cb))
            == ql.lib.qlinear_weights_bytes(1920, 1920, C.byref(cfg)) + 1920 * 1920 * 2)
    cq8 = ql.WeightCfg(ql.QL_W_QARVD_INT4, 0, 3.5, 2.0, 0, 1)                     # + int8 copy
    assert (ql.lib.qlinear_weights_bytes(384, 640, C.byref(cq8))
            == ql.lib.qlinear_weights_bytes(384, 640, C.byref(cq)) + 384 * 672)    # Kp = 640 + 32
    assert ql.lib.qlinear_quantize_ws_bytes(10, 130, 0) == 0
    assert ql.lib.qlinear_route_ws_bytes(-1) == 0 and ql.lib.qlinear_route_ws_bytes(10) > 0


FAKE = 1 << 20        # a 256-aligned non-null address; never dereferenced


def test_forward_rejects_bad_arguments_without_a_device(ql):
    w = ql.Weights(fmt=ql.QL_W_NVFP4, N=1920, K=1920, hadamard=1, codes=FAKE, sf=FAKE, gscale=FAKE)
    f = ql.lib.qlinear_forward
    assert f(None, 10, C.byref(w), 0, FAKE, FAKE, 1 << 30, None) == 1             # null X
    assert f(FAKE, -1, C.byref(w), 0, FAKE, FAKE, 1 << 30, None) == 1             # M < 0
    assert f(FAKE + 8, 10, C.byref(w), 0, FAKE, FAKE, 1 << 30, None) == 3         # misaligned X
    assert f(FAKE, 10, C.byref(w), 7, FAKE, FAKE, 1 << 30, None) == 1             # bad route
    assert f(FAKE, 10, C.byref(w), 0, FAKE, FAKE, 16, None) == 6                  # workspace
    bad = ql.Weights(fmt=ql.QL_W_NVFP4, N=1920, K=1000, hadamard=1, codes=FAKE, sf=FAKE, gscale=FAKE)
    assert f(FAKE, 10, C.byref(bad), 0, FAKE, FAKE, 1 << 30, None) == 2           # K % 128
    odd = ql.Weights(fmt=ql.QL_W_NVFP4, N=100, K=1920, hadamard=1, codes=FAKE, sf=FAKE, gscale=FAKE)
    assert f(FAKE, 10, C.byref(odd), 0, FAKE, FAKE, 1 << 30, None) == 2           # N % 16


def test_other_entry_points_reject_bad_arguments(ql):
    L = ql.lib
    assert L.qlinear_route(FAKE, FAKE, 100, 0.05, None, FAKE, FAKE, 1 << 20, None) == 1
    assert L.qlinear_route(FAKE + 4, FAKE, 100, 0.05, FAKE, FAKE, FAKE, 1 << 20, None) == 3
    assert L.qlinear_route(FAKE, FAKE, 100, 0.05, FAKE, FAKE, FAKE, 8, None) == 6
    assert L.qlinear_route(FAKE, FAKE, 100, float("nan"), FAKE, FAKE, FAKE, 1 << 20, None) == 1
    # token-split router
    assert L.qlinear_gamma_sums(FAKE, FAKE, 100, None, FAKE, 1 << 20, None) == 1
    assert L.qlinear_gamma_sums(FAKE, FAKE, -1, FAKE, FAKE, 1 << 20, None) == 1
    assert L.qlinear_gamma_sums(FAKE, FAKE + 8, 100, FAKE, FAKE, 1 << 20, None) == 3
    assert L.qlinear_gamma_sums(FAKE, FAKE, 100, FAKE + 4, FAKE, 1 << 20, None) == 3
    assert L.qlinear_gamma_sums(FAKE, FAKE, 100, FAKE, FAKE, 8, None) == 6
    assert L.qlinear_route_from_sums(None, 0.05, FAKE, FAKE, None) == 1
    assert L.qlinear_route_from_sums(FAKE, float("nan"), FAKE, FAKE, None) == 1
    assert L.qlinear_route_from_sums(FAKE, 0.05, FAKE + 4, FAKE, None) == 3
    na = L.qlinear_route_noalloc
    na.restype = C.c_int
    na.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p]
    assert na(FAKE, FAKE, -5, 0.05, FAKE, FAKE, None) == 1
    assert na(FAKE, FAKE + 2, 5, 0.05, FAKE, FAKE, None) == 3
    assert L.qlinear_tensor_amax(FAKE, 4, 96, 1, FAKE, FAKE, 1 << 20, None) == 2
    assert L.qlinear_quantize_act(FAKE, 4, 128, 9, 1, None, None, FAKE, FAKE, None, FAKE, FAKE,
                                  1 << 20, None) == 1
    cfg = ql.WeightCfg(ql.QL_W_QARVD_INT4, 1, 3.5, 2.0)                          # Q-ARVD has no rotation
    desc = ql.Weights()
    assert L.qlinear_prepare_weights(FAKE, 256, 256, C.byref(cfg), FAKE, 1 << 30, C.byref(desc),
                                     FAKE, 1 << 30, None) == 1
    for bad in (ql.WeightCfg(ql.QL_W_NVFP4, 1, 3.5, 2.0, 0, 1),                  # int8 copy of NVFP4
                ql.WeightCfg(ql.QL_W_QARVD_INT4, 0, 3.5, 2.0, 1, 0)):            # f16 copy of Q-ARVD
        assert L.qlinear_prepare_weights(FAKE, 256, 256, C.byref(bad), FAKE, 1 << 30, C.byref(desc),
                                         FAKE, 1 << 30, None) == 1
    assert L.qlinear_gemm(0, FAKE, FAKE, FAKE, 10, None, FAKE, None) == 1


def test_gemm_tile_count_limit(ql):
    """ceil(M/128) * ceil(N/128) must stay below 2^31: at the limit the GEMM
    entry points refuse the shape before anything else."""
    import torch
    L = ql.lib
    w = ql.Weights(fmt=ql.QL_W_NVFP4, N=1 << 22, K=128, hadamard=1, codes=FAKE, sf=FAKE, gscale=FAKE)
    m_over = (1 << 16) * 128                      # 2^16 x 2^15 tiles = 2^31
    assert L.qlinear_gemm(0, FAKE, FAKE, FAKE, m_over, C.byref(w), FAKE, None) == 2
    assert L.qlinear_forward(FAKE, m_over, C.byref(w), 0, FAKE, FAKE, 1 << 62, None) == 2
    assert L.qlinear_forward_routed(FAKE, m_over, C.byref(w), FAKE, FAKE, FAKE, 1 << 62, None) == 2
    if not torch.cuda.is_available():             # one tile row less passes every check but the device
        m_under = m_over - 128
        assert L.qlinear_gemm(0, FAKE, FAKE, FAKE, m_under, C.byref(w), FAKE, None) == 7
        assert L.qlinear_forward(FAKE, m_under, C.byref(w), 0, FAKE, FAKE, 1 << 62, None) == 7


def test_streaming_size_limit(ql):
    """M * K < 2^37: the streaming kernels read the input as 128-byte TMA rows
    with 32-bit row coordinates (2^20 x 2^17 passes the block-count rule)."""
    L = ql.lib
    assert L.qlinear_tensor_amax(FAKE, 1 << 20, 1 << 17, 1, FAKE, FAKE, 1 << 62, None) == 2
    assert L.qlinear_quantize_act(FAKE, 1 << 20, 1 << 17, 0, 1, None, None, FAKE, FAKE, None, FAKE, FAKE,
                                  1 << 62, None) == 2


def test_valid_call_without_a_device_reports_no_device(ql):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    w = ql.Weights(fmt=ql.QL_W_NVFP4, N=1920, K=1920, hadamard=1, codes=FAKE, sf=FAKE, gscale=FAKE)
    assert ql.lib.qlinear_forward(FAKE, 10, C.byref(w), 0, FAKE, FAKE, 1 << 30, None) == 7



def test_new_entry_points_validate_on_the_host(ql):
    """TDC, BF16 route, INT6 and decomposition arguments are checked before
    any CUDA call (no device needed)."""
    L = ql.lib
    prm = ql.TdcParams(0.05, 0.1, 0.3, 3, 8.0, 1.0)
    assert L.qlinear_tdc_init(None, None) == 1
    assert L.qlinear_tdc_init(FAKE + 4, None) == 3                                   # state not 8-aligned
    assert L.qlinear_tdc_refresh(FAKE, FAKE, 100, FAKE, FAKE, None, C.byref(prm), FAKE, 1 << 20, None) == 1
    assert L.qlinear_tdc_refresh(FAKE, FAKE, 100, FAKE, FAKE + 8, FAKE, C.byref(prm), FAKE, 1 << 20, None) == 3
    assert L.qlinear_tdc_refresh(FAKE, FAKE, 100, FAKE, FAKE, FAKE, C.byref(prm), FAKE, 16, None) == 6
    for fields in [(0.05, float("nan"), 0.3, 3, 8.0, 1.0), (0.05, 0.1, 0.3, 3, float("nan"), 1.0),
                   (0.05, 0.1, 0.3, 3, 8.0, float("nan"))]:
        nan = ql.TdcParams(*fields)
        assert L.qlinear_tdc_refresh(FAKE, FAKE, 100, FAKE, FAKE, FAKE, C.byref(nan), FAKE, 1 << 20, None) == 1
        assert L.qlinear_tdc_skip(FAKE, 100, FAKE, FAKE, FAKE, C.byref(nan), FAKE, None) == 1
    neg = ql.TdcParams(0.05, 0.1, 0.3, -1, 8.0, 1.0)
    assert L.qlinear_tdc_skip(FAKE, 100, FAKE, FAKE, FAKE, C.byref(neg), FAKE, None) == 1
    assert L.qlinear_tdc_skip(FAKE, 100, FAKE, FAKE, FAKE, None, FAKE, None) == 1
    assert L.qlinear_tdc_ws_bytes(-1) == 0 and L.qlinear_tdc_ws_bytes(1000) > 0
    # the BF16 route needs kept bf16 weights; other formats reject it
    w = ql.Weights(fmt=ql.QL_W_NVFP4, N=1920, K=1920, hadamard=1, codes=FAKE, sf=FAKE, gscale=FAKE)
    assert L.qlinear_gemm(ql.QL_ROUTE_BF16, FAKE, None, None, 10, C.byref(w), FAKE, None) == 1
    assert L.qlinear_forward_ws_bytes(10, C.byref(w), ql.QL_ROUTE_BF16) == 0
    wq = ql.Weights(fmt=ql.QL_W_QARVD_INT4, N=256, K=256, codes=FAKE, Kp=256 + 32, gather=FAKE, kinfo=FAKE,
                    s_norm=FAKE, s_out=FAKE)
    assert L.qlinear_gemm(ql.QL_ROUTE_BF16, FAKE, None, None, 10, C.byref(wq), FAKE, None) == 1
    # INT6 formats size like their INT8 counterparts; unknown formats size to 0
    assert L.qlinear_quantize_ws_bytes(10, 256, ql.QL_ROUTE_INT6) == L.qlinear_quantize_ws_bytes(10, 256, ql.QL_ROUTE_INT8)
    assert L.qlinear_quantize_ws_bytes(10, 256, ql.QL_ACT_INT6_TENSOR) > 0
    assert L.qlinear_quantize_ws_bytes(10, 256, 99) == 0
    # decomposed weights: twice the codes, scales over 2K; not with an f16 or bf16 copy
    cd = ql.WeightCfg(ql.QL_W_NVFP4_DECOMP, 1, 3.5, 2.0)
    cn = ql.WeightCfg(ql.QL_W_NVFP4, 1, 3.5, 2.0)
    assert L.qlinear_weights_bytes(640, 1920, C.byref(cd)) > L.qlinear_weights_bytes(640, 1920, C.byref(cn))
    desc = ql.Weights()
    for bad in (ql.WeightCfg(ql.QL_W_NVFP4_DECOMP, 1, 3.5, 2.0, 1, 0, 0), ql.WeightCfg(ql.QL_W_NVFP4_DECOMP, 1, 3.5, 2.0, 0, 0, 1)):
        assert L.qlinear_prepare_weights(FAKE, 256, 256, C.byref(bad), FAKE, 1 << 30, C.byref(desc),
                                         FAKE, 1 << 30, None) == 1
    # decomposed weights run the decomposed NVFP4 route only
    wd = ql.Weights(fmt=ql.QL_W_NVFP4_DECOMP, N=1920, K=1920, hadamard=1, codes=FAKE, sf=FAKE, gscale=FAKE)
    assert L.qlinear_forward_ws_bytes(10, C.byref(wd), ql.QL_ROUTE_INT8) == 0
    assert L.qlinear_forward(FAKE, 10, C.byref(wd), ql.QL_ROUTE_INT8, FAKE, FAKE, 1 << 30, None) == 1
    # the division test hook
    assert L.qlinear_debug_div_check(0.0, 0, 10, FAKE, None) == 1
    assert L.qlinear_debug_div_check(1.0, 0x7F800000, 1, FAKE, None) == 1
    assert L.qlinear_debug_div_check(1.0, 0, 10, None, None) == 1
