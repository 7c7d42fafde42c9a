"""Parity of the split-KV decode entry point with the fp64 oracle."""
import pytest
import torch

import oracle
import workloads
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
    d = to_dev(p)
    o, l = run(p, d, "decode", num_splits=num_splits)
    torch.cuda.synchronize()
    if pairs is None:
        ro, rl = oracle.problem(p)
        return compare(o, l, ro, rl, p.q.dtype, p.name), (o, l)
    ro, rl = oracle.problem(p, pairs=pairs)
    return compare(o.cpu()[pairs[:, 0], pairs[:, 1]], l.cpu()[pairs[:, 0], pairs[:, 1]], ro, rl, p.q.dtype,
                   p.name), (o, l)


@pytest.mark.parametrize("splits", [0, 1, 2, 3, 8])
def test_mla_small(splits):
    p = workloads.mla_decode(21, batch=3, q_len=4, kv_len=700)
    check(p, splits)


def test_mla_ragged_lengths():
    p = workloads.mla_decode(22, batch=5, q_len=4, kv_len=0, lens_kv=[1, 64, 65, 1000, 129])
    check(p)


def test_mla_one_long_sequence():
    # 625 KV tiles of one sequence cut at every CTA boundary: every piece of
    # the automatic schedule starts at a distinct cut inside the sequence
    p = workloads.mla_decode(25, batch=1, q_len=4, kv_len=40000)
    check(p)


def test_mla_cuts_on_sequence_starts():
    # 4 x 37 = 148 tiles of 64 keys over 148 CTAs: the cuts fall on every tile
    # boundary, three of them on sequence starts (not cuts inside a sequence)
    p = workloads.mla_decode(26, batch=4, q_len=4, kv_len=37 * 64)
    check(p)


def test_mla_fewer_tiles_than_ctas():
    # 128 tiles for 148 CTAs: several cut values repeat (empty CTA ranges)
    p = workloads.mla_decode(27, batch=1, q_len=4, kv_len=8192)
    check(p)


def test_mla_empty_sequences_single_launch():
    # a small problem (one-launch schedule) with sequences that have no key
    p = workloads.mla_decode(28, batch=4, q_len=4, kv_len=0, lens_kv=[0, 100, 0, 700])
    check(p)


def test_mla_single_launch_matches_split_schedule():
    # the same small problem through the one-launch schedule (automatic) and
    # through the prep + decode + combine schedule (fixed split count)
    p = workloads.mla_decode(29, batch=2, q_len=4, kv_len=3000)
    _, (o0, l0) = check(p, 0)
    _, (o5, l5) = check(p, 5)
    assert (o0.float() - o5.float()).abs().max() <= 4e-3
    assert (l0 - l5).abs().max() <= 1e-4


def test_mla_fp16_and_small_q():
    p = workloads.mla_decode(23, batch=4, q_len=1, kv_len=333, dtype="f16")
    check(p)


def test_mla_split_invariance():
    p = workloads.mla_decode(24, batch=2, q_len=4, kv_len=2048)
    _, (o1, l1) = check(p, 1)
    _, (o8, l8) = check(p, 8)
    assert (o1.float() - o8.float()).abs().max() <= 4e-3
    assert (l1 - l8).abs().max() <= 1e-4


@pytest.mark.parametrize("dims,dt", [((128, 128), "bf16"), ((64, 64), "f16"), ((128, 128), "f32")])
def test_gqa_decode(dims, dt):
    dqk, dv = dims
    p = workloads.varlen(25, [1, 1, 2, 1], [300, 1, 77, 1024], 8, 2, dqk, dt, False)
    d = to_dev(p)
    o, l = run(p, d, "decode")
    ro, rl = oracle.problem(p)
    compare(o, l, ro, rl, p.q.dtype, "gqa decode")


def test_full_size_mla_sampled():
    p = workloads.cfg_mla_decode()
    pairs = workloads.sample_rows(p, 16, 104)
    check(p, 0, pairs)


# ---------------------------------------------------------------- grouped-query decode on the tensor cores
@pytest.mark.parametrize("splits", [0, 1, 3, 8])
def test_gqa_tc_small(splits):
    p = workloads.gqa_decode(31, batch=3, q_len=1, kv_len=700)
    check(p, splits)


def test_gqa_tc_ragged_and_empty_lengths():
    # a sequence without keys ends at O = 0, LSE = -inf (written by the combine pass)
    p = workloads.gqa_decode(32, batch=6, q_len=1, kv_len=0, lens_kv=[1, 64, 65, 1000, 0, 129])
    check(p)
    check(p, 2)


@pytest.mark.parametrize("q_len,causal", [(4, True), (4, False), (8, True)])
def test_gqa_tc_several_queries(q_len, causal):
    # q_len * G rows per KV head: 32, 32 and 64 (the largest the kernel takes)
    p = workloads.gqa_decode(33, batch=3, q_len=q_len, kv_len=333, causal=causal)
    check(p)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_gqa_tc_d64(dt):
    p = workloads.gqa_decode(34, batch=4, q_len=2, kv_len=517, hq=16, hkv=2, d=64, dtype=dt)
    check(p)
    check(p, 3)


def test_gqa_tc_group_sizes():
    # G = 1 (one query head per KV head) and G = 16
    check(workloads.gqa_decode(35, batch=2, q_len=1, kv_len=300, hq=8, hkv=8))
    check(workloads.gqa_decode(36, batch=2, q_len=2, kv_len=300, hq=32, hkv=2))


def test_gqa_rows_beyond_tensor_core_limit():
    # more than 64 queries per sequence: the exact CUDA-core kernel takes it
    check(workloads.gqa_decode(37, batch=2, q_len=70, kv_len=200, hq=4, hkv=4, causal=True))


@pytest.mark.parametrize("q_len,hq,hkv,causal", [(16, 32, 4, True), (4, 32, 1, False), (3, 48, 2, True),
                                                 (64, 8, 4, True)])
def test_gqa_tc_head_groups(q_len, hq, hkv, causal):
    # q_len * Hq/Hkv = 128, 128, 72 and 128 rows per KV head: the query heads
    # of each KV head split into two groups (of 4, 16, 12 and 1 heads) on the
    # tensor cores
    p = workloads.gqa_decode(39, batch=3, q_len=q_len, kv_len=700, hq=hq, hkv=hkv, causal=causal)
    check(p)
    check(p, 3)


@pytest.mark.parametrize("batch,kv_len,splits", [(3, 700, 0), (3, 700, 2), (2, 40000, 0), (200, 300, 0)])
def test_mla_q8_head_groups(batch, kv_len, splits):
    # 8 queries x 16 heads = 128 query rows: two groups of 8 heads, each
    # streaming the latent cache; one launch (small), three kernels (a long
    # sequence, or more sequences than SMs)
    p = workloads.mla_decode(29, batch=batch, q_len=8, kv_len=kv_len)
    if batch * 8 * 16 * kv_len > 50_000_000:
        check(p, splits, workloads.sample_rows(p, 8, 7))
    else:
        check(p, splits)


def test_gqa_tc_split_invariance():
    p = workloads.gqa_decode(38, batch=2, q_len=1, kv_len=4096)
    _, (o1, l1) = check(p, 1)
    _, (o8, l8) = check(p, 8)
    assert (o1.float() - o8.float()).abs().max() <= 4e-3
    assert (l1 - l8).abs().max() <= 1e-4


def test_full_size_gqa_sampled():
    p = workloads.cfg_gqa_decode()
    pairs = workloads.sample_rows(p, 16, 105)
    check(p, 0, pairs)
