"""Parity of the fp8-KV MLA decode entry point (mxfa_attn_decode_mla_fp8kv)
with the fp64 oracle over the dequantised cache."""
import pytest
import torch

import oracle
import workloads
from oracle import e4m3
from parity import compare
from runners import run, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import tiled_attention_21_b200 as mx
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mx.load()


def check(p, num_splits=0, pairs=None):
    import tiled_attention_21_b200 as mx
    d = to_dev(p)
    o, l = run(p, d, "decode", num_splits=num_splits)
    torch.cuda.synchronize()
    assert mx.read_device_status()[0] == 0
    if pairs is None:
        ro, rl = oracle.problem(p)
        return compare(o, l, ro, rl, p.q.dtype, p.name)
    ro, rl = oracle.problem(p, pairs=pairs)
    return compare(o.cpu()[pairs[:, 0], pairs[:, 1]], l.cpu()[pairs[:, 0], pairs[:, 1]], ro, rl, p.q.dtype, p.name)


def _all_codes_row():
    """576 codes holding every finite E4M3 code in the value columns: columns
    0-255 count up, 256-511 count down (NaN codes 0x7f / 0xff replaced by
    their finite neighbours), 512-575 repeat 0x00..0x3f."""
    up = torch.arange(256, dtype=torch.int32)
    up[0x7F], up[0xFF] = 0x7E, 0xFE
    row = torch.cat([up, up.flip(0), torch.arange(64, dtype=torch.int32)])
    return row.to(torch.uint8)


@pytest.mark.parametrize("kv_len,splits", [(1, 0), (128, 0), (128, 2), (8192, 0), (8192, 5)])
def test_every_code_widens_exactly(kv_len, splits):
    """Every key of a sequence holds the same row, so every score is equal,
    every probability is exactly 1 and O is exactly kv_scale times the value
    row: the widening of each of the 254 finite codes, the output scale on
    the direct store, on the partials and through the merge, all bit-exact.
    (kv_len 8192 with automatic splits runs the one-launch merge; splits = 5
    the partial + combine kernels.)"""
    p = workloads.mla_decode_fp8(41, batch=2, q_len=4, kv_len=kv_len)
    p.kv[:] = _all_codes_row()
    p.kv_scale = 0.5  # a power of two: kv_scale * value is exact in bf16
    d = to_dev(p)
    o, l = run(p, d, "decode", num_splits=splits)
    torch.cuda.synchronize()
    want = (e4m3.decode(_all_codes_row()[:512]) * 0.5).float()
    got = o.float().cpu()
    assert torch.equal(got, want.expand_as(got)), (got - want).abs().max()
    ro, rl = oracle.problem(p)
    compare(o, l, ro, rl, p.q.dtype, p.name)


@pytest.mark.parametrize("splits", [0, 1, 3, 8])
def test_fp8_small(splits):
    check(workloads.mla_decode_fp8(42, batch=3, q_len=4, kv_len=700), splits)


def test_fp8_ragged_and_empty_sequences():
    check(workloads.mla_decode_fp8(43, batch=6, q_len=4, kv_len=0, lens_kv=[1, 0, 65, 1000, 0, 129]))


def test_fp8_causal_q4():
    check(workloads.mla_decode_fp8(44, batch=4, q_len=4, kv_len=0, lens_kv=[3, 64, 300, 2000], causal=True))


def test_fp8_one_long_sequence():
    check(workloads.mla_decode_fp8(45, batch=1, q_len=4, kv_len=40000))


def test_fp8_three_kernel_path():
    # 64 x 32 tiles > 4 per SM: schedule, decode and combine kernels
    check(workloads.mla_decode_fp8(46, batch=64, q_len=4, kv_len=2048))


def test_fp8_scale_and_softmax_scale():
    # A negative scale flips every score and every output.  Its magnitude is
    # the workload's own, so the dequantised values keep unit scale, which
    # the absolute 1e-2 bound assumes (bf16 rounding of P, 2^-9 relative,
    # times |v|).
    p = workloads.mla_decode_fp8(47, batch=3, q_len=2, kv_len=777)
    p.kv_scale = -p.kv_scale
    p.scale = 0.05
    check(p)


def test_fp8_full_size_sampled_rows():
    """The benchmarked shape (batch 128, q_len 4, 16 heads, kv 8192) in the
    launch configuration bench.py times, checked on sampled rows."""
    p = workloads.cfg_mla_decode_fp8()
    pairs = workloads.sample_rows(p, 2, 5)
    check(p, pairs=pairs)


def test_fp8_rejects_unsupported_shapes():
    import tiled_attention_21_b200 as mx
    p = workloads.mla_decode_fp8(48, batch=2, q_len=8, kv_len=64, heads=16)  # 128 query rows
    d = to_dev(p)
    with pytest.raises(mx.MxfaError) as e:
        run(p, d, "decode")
    assert e.value.status == mx.MXFA_ERR_UNSUPPORTED
