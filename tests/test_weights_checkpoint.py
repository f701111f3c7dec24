"""Checkpoint of packed weights on the host: state_dict() records each
descriptor array as an offset into the weight buffer, and from_state_dict()
rebases every pointer onto a new buffer.  Exercised here with a CPU buffer
standing in for the device one (the bookkeeping is the same)."""
import io

import pytest
import torch


@pytest.fixture(scope="module")
def ql():
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


def test_field_lists_cover_the_descriptor(ql):
    fields = {f for f, _ in ql.Weights._fields_}
    assert set(ql._WEIGHT_SIZES) | set(ql._WEIGHT_ARRAYS) | {"reserved0"} == fields
    assert not set(ql._WEIGHT_SIZES) & set(ql._WEIGHT_ARRAYS)


def _fake(ql):
    buf = torch.arange(4096, dtype=torch.int64).to(torch.uint8)
    base = buf.data_ptr()
    desc = ql.Weights(fmt=ql.QL_W_QARVD_INT4, N=64, K=256, hadamard=0, Kp=288)
    offs = dict(codes=0, gather=1024, kinfo=2048, s_norm=2304, s_out=2560, norms=2816, perm=3328,
                outlier_mask=3840, w8=None, sf=None, gscale=None, w16=None, wbf16=None)
    for f, o in offs.items():
        setattr(desc, f, None if o is None else base + o)
    return ql.PackedWeights(desc, buf, 64, 256, ql.QL_W_QARVD_INT4), offs


def test_round_trip_through_torch_save(ql):
    pw, offs = _fake(ql)
    sd = pw.state_dict()
    assert sd["offsets"] == offs
    f = io.BytesIO()
    torch.save(sd, f)
    f.seek(0)
    pw2 = ql.PackedWeights.from_state_dict(torch.load(f), "cpu")
    assert torch.equal(pw2.buf, pw.buf) and pw2.buf.data_ptr() != pw.buf.data_ptr()
    base2 = pw2.buf.data_ptr()
    for name, o in offs.items():
        assert getattr(pw2.desc, name) == (None if o is None else base2 + o), name
    for name in ql._WEIGHT_SIZES:
        assert getattr(pw2.desc, name) == getattr(pw.desc, name)
    assert (pw2.N, pw2.K, pw2.fmt) == (64, 256, ql.QL_W_QARVD_INT4)


def test_bad_checkpoints_are_rejected(ql):
    pw, _ = _fake(ql)
    sd = pw.state_dict()
    with pytest.raises(ValueError, match="ABI"):
        ql.PackedWeights.from_state_dict(dict(sd, abi=sd["abi"] - 1), "cpu")
    with pytest.raises(ValueError, match="outside"):
        ql.PackedWeights.from_state_dict(dict(sd, offsets=dict(sd["offsets"], codes=4096)), "cpu")
    with pytest.raises(TypeError):
        ql.PackedWeights.from_state_dict(dict(sd, buf=sd["buf"].float()), "cpu")
    pw.desc.codes = pw.buf.data_ptr() + 5000          # an array outside the buffer
    with pytest.raises(ValueError, match="does not point"):
        pw.state_dict()
