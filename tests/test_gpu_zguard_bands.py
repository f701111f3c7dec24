"""Out-of-bounds write check (guard bands): every route's output Y, and the
TDC skip output, is placed inside a larger buffer whose margins hold a
canary pattern.  After the call the margins must be unchanged and Y must
equal the output of the same call into a buffer of its own.  The shapes
are ragged (M not a multiple of 128, N not a multiple of the tile width)
so that the last tiles are partial.  The same prepared weights also go
through a checkpoint (state_dict, torch.save, from_state_dict) and must
give the identical forward."""
import pytest
import torch

from bit_quantized_linear_block_b200 import synthetic as S

pytestmark = pytest.mark.gpu

PAD = 4096          # bf16 elements on each side (8 KB: keeps Y 256-byte aligned)
CANARY = -7.5


@pytest.fixture(scope="module")
def ql():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


def _guarded(rows, cols):
    big = torch.full((PAD + rows * cols + PAD,), CANARY, dtype=torch.bfloat16, device="cuda")
    return big, big[PAD:PAD + rows * cols].view(rows, cols)


def _margins_intact(big, n):
    return bool((big[:PAD] == CANARY).all()) and bool((big[PAD + n:] == CANARY).all())


def _prepare(ql, kind, n, k, seed):
    if kind.startswith("qarvd"):
        w = S.weights(n, k, 0.02, seed, 77, outlier_frac=0.05, outlier_scale=20.0)
        return ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_QARVD_INT4, hadamard=False,
                                          expand_i8=kind.endswith("copy"))
    w = S.weights(n, k, 0.02, 7, seed)
    if kind == "decomp":
        return ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4_DECOMP, hadamard=True)
    return ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True,
                                      expand_f16=kind.endswith("copy"), keep_bf16=(kind == "bf16"))


CASES = [  # (kind, route, m, n, k)
    ("nvfp4", 0, 300, 1040, 640),          # ragged 192-wide tiles, CTA pairs
    ("nvfp4", 0, 100, 1040, 2048),         # one SM per tile, streamed scales
    ("int8", 1, 300, 384, 640),            # FP4 weights widened on chip
    ("int8_copy", 1, 300, 384, 640),       # f16 weight copy
    ("int6_copy", 5, 129, 640, 384),
    ("bf16", 8, 300, 384, 640),
    ("qarvd", 2, 300, 384, 640),           # INT4 widened on chip
    ("qarvd_copy", 2, 300, 384, 640),      # int8 weight copy, CTA pairs
    ("decomp", 0, 129, 640, 384),
]


@pytest.mark.parametrize("kind,route,m,n,k", CASES)
def test_forward_writes_only_its_output(ql, kind, route, m, n, k):
    x = S.activations_fixed_outliers(m, k, 8, 50.0, m + n, 1).cuda()
    pw = _prepare(ql, kind, n, k, m + n + k)
    y_plain = ql.qlinear_forward(x, pw, route)
    big, y = _guarded(m, n)
    ql.qlinear_forward(x, pw, route, Y=y)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert _margins_intact(big, m * n)
    assert torch.equal(y, y_plain)


def test_tdc_skip_writes_only_its_output(ql):
    numel = 1001                            # ragged: not a multiple of the 8-element vectors
    x, y, _ = S.dmpq_block_pair(1, m=1, k=1920)
    inp, out = x.reshape(-1)[:numel].contiguous().cuda(), y.reshape(-1)[:numel].contiguous().cuda()
    cache = ql.TdcCache(numel, "cuda")
    ql.qlinear_tdc_refresh(inp, out, cache)
    plain = ql.qlinear_tdc_skip(inp, cache)
    big, guarded = _guarded(1, numel)
    ql.qlinear_tdc_skip(inp, cache, out=guarded.view(-1))
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert _margins_intact(big, numel)
    assert torch.equal(guarded.view(-1), plain)


@pytest.mark.parametrize("kind,route,m,n,k", [CASES[0], CASES[3], CASES[5], CASES[7], CASES[8]])
def test_checkpointed_weights_give_the_same_output(ql, kind, route, m, n, k):
    """Packed weights saved with torch.save(pw.state_dict()) and reloaded onto
    the device produce the identical forward, with the original buffer
    zeroed (the weight buffer holds no addresses)."""
    import io
    x = S.activations_fixed_outliers(m, k, 8, 50.0, m + n, 1).cuda()
    pw = _prepare(ql, kind, n, k, m + n + k)
    y0 = ql.qlinear_forward(x, pw, route)
    f = io.BytesIO()
    torch.save(pw.state_dict(), f)
    f.seek(0)
    pw2 = ql.PackedWeights.from_state_dict(torch.load(f), "cuda")
    pw.buf.zero_()        # the reloaded weights must not read the original buffer
    y1 = ql.qlinear_forward(x, pw2, route)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert torch.equal(y0, y1)
