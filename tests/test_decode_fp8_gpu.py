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
    p = workloads.mla_decode_fp8(48, batch=2, q_len=65, kv_len=64, heads=2)  # more than 64 queries
    d = to_dev(p)
    with pytest.raises(mx.MxfaError) as e:
        run(p, d, "decode")
    assert e.value.status == mx.MXFA_ERR_UNSUPPORTED


@pytest.mark.parametrize("kv_len,splits", [(300, 0), (300, 3), (8192, 0)])
def test_fp8_q8_head_groups(kv_len, splits):
    # 8 queries x 16 heads = 128 query rows: two groups of 8 heads on the tensor cores
    p = workloads.mla_decode_fp8(49, batch=3, q_len=8, kv_len=kv_len, causal=True)
    check(p, splits)


def test_fp8_padded_cache_rows():
    """Cache rows 640 bytes apart (576 codes + padding): the row stride is an
    argument, and the padding is never read."""
    import tiled_attention_21_b200 as mx
    p = workloads.mla_decode_fp8(49, batch=3, q_len=4, kv_len=0, lens_kv=[700, 65, 1300])
    d = to_dev(p)
    padded = torch.full((p.total_k, 640), 0x7E, dtype=torch.uint8, device="cuda")  # padding: 448
    padded[:, :576] = d["kv"]
    o, l = mx.mxfa_attn_decode_mla_fp8kv(d["q"], padded[:, :576], p.kv_scale, d["cu_q"], d["cu_k"], 4, 1300,
                                         softmax_scale=p.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.problem(p)
    compare(o, l, ro, rl, p.q.dtype, p.name)


def test_fp8_all_sequences_empty():
    """total_kv = 0 with a valid, never-read cache pointer (the C entry point
    directly: torch hands out no pointer for an empty tensor): O = 0 and
    LSE = -inf."""
    import tiled_attention_21_b200 as mx
    lib = mx.load()
    q = torch.randn(8, 16, 576, device="cuda").to(torch.bfloat16)
    cu_q = torch.tensor([0, 4, 8], dtype=torch.int32, device="cuda")
    cu_k = torch.zeros(3, dtype=torch.int32, device="cuda")
    kv = torch.zeros(1, 576, dtype=torch.uint8, device="cuda")
    o = torch.full((8, 16, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    l = torch.zeros(8, 16, dtype=torch.float32, device="cuda")
    need = lib.mxfa_attn_decode_mla_fp8kv_workspace_size(2, 4, 16, 0, 0)
    ws = mx.workspace(need, q.device)
    wp, wn = mx._ws_view(ws)
    st = lib.mxfa_attn_decode_mla_fp8kv(q.data_ptr(), kv.data_ptr(), 0.5, o.data_ptr(), l.data_ptr(),
                                        cu_q.data_ptr(), cu_k.data_ptr(), 2, 8, 0, 4, 0, 16, 576, float("nan"), 0, 0,
                                        wp, wn, mx._stream(None))
    assert st == mx.MXFA_OK, lib.mxfa_last_error()
    torch.cuda.synchronize()
    assert mx.read_device_status()[0] == 0
    assert torch.equal(o.float().cpu(), torch.zeros(8, 16, 512))
    assert bool(torch.isinf(l).all() and (l < 0).all())
