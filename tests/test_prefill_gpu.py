"""Parity of the prefill entry points (batched and varlen) with the fp64 oracle."""
import math

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


def check_full(p, entry=None):
    d = to_dev(p)
    o, l = run(p, d, entry)
    torch.cuda.synchronize()
    ro, rl = oracle.problem(p)
    return compare(o, l, ro, rl, p.q.dtype, p.name)


def test_single_head_fp32():
    check_full(workloads.cfg_single_head_fp32())


BATCHED = [
    # (B, Sq, Sk, Hq, Hkv, D, dtype, causal)
    (1, 128, 128, 1, 1, 128, "bf16", False),
    (2, 300, 300, 4, 4, 128, "bf16", True),
    (2, 300, 300, 4, 4, 128, "bf16", False),
    (1, 513, 513, 8, 2, 128, "bf16", True),
    (2, 200, 333, 4, 2, 128, "bf16", True),    # Sq < Sk: bottom-right diagonal
    (1, 333, 200, 2, 1, 128, "bf16", True),    # Sq > Sk: first rows see nothing
    (2, 257, 129, 4, 1, 64, "bf16", True),
    (1, 700, 700, 2, 2, 64, "f16", True),
    (2, 384, 384, 4, 2, 128, "f16", False),
    (1, 1, 1, 2, 2, 128, "bf16", True),
    (1, 77, 1000, 2, 2, 128, "bf16", False),
    (2, 96, 96, 4, 2, 64, "f32", True),
    (1, 130, 250, 4, 4, 128, "f32", False),
]


@pytest.mark.parametrize("case", BATCHED, ids=lambda c: "b{}_sq{}_sk{}_h{}x{}_d{}_{}_{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], c[6], "causal" if c[7] else "full"))
def test_batched(case):
    B, Sq, Sk, Hq, Hkv, D, dt, causal = case
    check_full(workloads.batched(11, B, Sq, Sk, Hq, Hkv, D, dt, causal))


VARLEN = [
    ([1, 130, 257, 600, 5], [1, 130, 257, 600, 5], 8, 2, 128, "bf16", True),
    ([300, 0, 17, 512], [300, 9, 40, 512], 4, 4, 128, "bf16", True),
    ([64, 200, 129], [70, 10, 400], 4, 1, 64, "f16", False),
    ([100, 50], [0, 80], 2, 2, 128, "bf16", True),  # a sequence without keys
    ([33, 1, 65], [40, 1, 65], 4, 2, 128, "f32", True),
]


@pytest.mark.parametrize("case", VARLEN, ids=lambda c: f"{len(c[0])}seq_h{c[2]}x{c[3]}_d{c[4]}_{c[5]}")
def test_varlen(case):
    lq, lk, Hq, Hkv, D, dt, causal = case
    check_full(workloads.varlen(12, lq, lk, Hq, Hkv, D, dt, causal))


def test_batched_equals_varlen_entry():
    p = workloads.batched(13, 3, 260, 260, 4, 2, 128, "bf16", True)
    d = to_dev(p)
    o1, l1 = run(p, d, "fwd")
    o2, l2 = run(p, d, "varlen")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_strided_views():
    """q/k/v sliced out of one packed [B, S, 3, H, D] tensor (row stride 3*H*D)."""
    import tiled_attention_21_b200 as mx
    g = torch.Generator().manual_seed(5)
    B, S, H, D = 2, 300, 4, 128
    qkv = torch.randn(B, S, 3, H, D, generator=g).to(torch.bfloat16)
    q, k, v = (qkv[:, :, i] for i in range(3))
    o, l = mx.mxfa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    ro, rl = oracle.attention(q.reshape(B * S, H, D), k.reshape(B * S, H, D), v.reshape(B * S, H, D),
                              [0, S, 2 * S], [0, S, 2 * S], D ** -0.5, True)
    compare(o.view(B * S, H, D), l.view(B * S, H), ro, rl, torch.bfloat16, "strided")


def test_scale_zero_and_negative():
    for scale in (0.0, -0.2):
        p = workloads.batched(14, 1, 260, 260, 2, 2, 128, "bf16", True, scale=scale)
        check_full(p)


def test_negative_scale_masked_tiles():
    """A negative scale on the tensor-core path (the scores are negated in
    registers and |scale| is used): causal diagonal tiles, a ragged last
    tile, Sq != Sk, D = 64 and f16, and a varlen grouped-query batch.  The
    scales stay near head_dim^-0.5: at |scale| = 0.3 with D = 128 the
    softmax is so peaked that the oracle rounded to bf16 is already 0.8-1.2e-2
    from the oracle, beyond the 1e-2 bound for either sign."""
    check_full(workloads.batched(15, 2, 300, 300, 4, 2, 64, "f16", True, scale=-0.11))
    check_full(workloads.batched(15, 1, 200, 333, 4, 4, 128, "bf16", False, scale=-0.1))
    check_full(workloads.batched(15, 1, 333, 200, 2, 1, 128, "bf16", True, scale=-0.05))
    check_full(workloads.varlen(15, [129, 1, 300], [129, 7, 300], 8, 2, 128, "bf16", True, scale=-0.09))


def test_large_scores_x50():
    """q, k scaled by 50 (oxillama-runtime flash_attention.rs,
    test_flash_attention_numerical_stability): O finite and within tolerance.
    The scores are now ~1e3, so LSE carries the rounding of an fp32 sum of D
    products: its bound is 1e-3 plus D * 2^-24 * scale * max_j sum_d |q_d k_jd|
    (the worst-case error of that sum), per row."""
    p = workloads.batched(15, 1, 300, 300, 2, 2, 128, "bf16", True)
    p.q = (p.q.float() * 50).to(torch.bfloat16)
    p.k = (p.k.float() * 50).to(torch.bfloat16)
    d = to_dev(p)
    o, l = run(p, d)
    ro, rl = oracle.problem(p)
    qa, ka = p.q.double().abs(), p.k.double().abs()
    bound = torch.einsum("ihd,jhd->hij", qa, ka).amax(-1).transpose(0, 1) * p.scale
    compare(o, l, ro, rl, torch.bfloat16, "x50", lse_tol=1e-3 + 128 * 2.0 ** -24 * bound)


def test_position_code_indexing_exact():
    """q = 0: every visible score is 0, so exp(LSE) is the visible count
    (recovered exactly by rounding) and O is the mean of the visible v."""
    lq, lk = [1, 130, 257, 600, 5, 0, 300], [1, 130, 300, 600, 50, 7, 299]
    p = workloads.varlen(16, lq, lk, 8, 2, 128, "bf16", True)
    p.q = torch.zeros_like(p.q)
    v = torch.zeros_like(p.v, dtype=torch.float32)
    ck = p.cu_k.tolist()
    for b in range(len(lk)):
        j = torch.arange(lk[b], dtype=torch.float32)
        v[ck[b]:ck[b + 1], :, 0] = (j % 64)[:, None]
        v[ck[b]:ck[b + 1], :, 1] = (j // 64)[:, None]
    p.v = v.to(torch.bfloat16)
    d = to_dev(p)
    o, l = run(p, d)
    ro, rl = oracle.problem(p)
    fin = torch.isfinite(rl)
    count_gpu = torch.round(torch.exp(l.double().cpu()[fin]))
    count_ref = torch.round(torch.exp(rl[fin]))
    assert torch.equal(count_gpu, count_ref)
    assert torch.equal(torch.isfinite(l.cpu()), fin)
    compare(o, l, ro, rl, torch.bfloat16, "position code")


def test_deterministic():
    p = workloads.batched(17, 2, 600, 600, 4, 2, 128, "bf16", True)
    d = to_dev(p)
    o1, l1 = run(p, d)
    o2, l2 = run(p, d)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_causal_last_row_equals_full():
    p = workloads.batched(18, 1, 384, 384, 2, 2, 128, "bf16", True)
    d = to_dev(p)
    oc, lc = run(p, d)
    p.causal = False
    of, lf = run(p, d)
    assert (oc[-1].float() - of[-1].float()).abs().max() <= 2e-3
    assert (lc[-1] - lf[-1]).abs().max() <= 1e-4


def _sampled(p, n_per_head, seed):
    d = to_dev(p)
    o, l = run(p, d)
    torch.cuda.synchronize()
    pairs = p.check_rows if p.check_rows is not None else workloads.sample_rows(p, n_per_head, seed)
    ro, rl = oracle.problem(p, pairs=pairs)
    o_s = o.cpu()[pairs[:, 0], pairs[:, 1]]
    l_s = l.cpu()[pairs[:, 0], pairs[:, 1]]
    return compare(o_s, l_s, ro, rl, p.q.dtype, p.name)


def test_full_size_batched_causal_sampled():
    _sampled(workloads.cfg_batched_causal(), 48, 101)


def test_full_size_varlen_gqa_sampled():
    _sampled(workloads.cfg_varlen_gqa(), 24, 102)


def test_full_size_long_context_sampled():
    _sampled(workloads.cfg_long_causal(), 0, 103)


def test_varlen_max_seqlen_below_a_length_is_reported():
    """max_seqlen_q sizes the varlen schedule; a sequence longer than it
    leaves 256-row blocks unscheduled, which the schedule kernel reports as
    MXFA_ERR_INVALID_ARG at site 0x201 (strict mode off, so the host does not
    read cu_seqlens)."""
    import tiled_attention_21_b200 as mx
    p = workloads.varlen(19, [1000, 10], [1000, 10], 4, 4, 128, "bf16", True)
    d = to_dev(p)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    mx.mxfa_attn_varlen_fwd(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"], 300, 1000, causal=True, ws=ws)
    st, site = mx.read_device_status(ws)
    assert (st, site) == (mx.MXFA_ERR_INVALID_ARG, 0x201)
    # the status was cleared by the read; a call with the true maximum is clean
    o, l = mx.mxfa_attn_varlen_fwd(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"], 1000, 1000, causal=True, ws=ws)
    assert mx.read_device_status(ws)[0] == mx.MXFA_OK
    ro, rl = oracle.problem(p)
    compare(o, l, ro, rl, p.q.dtype, p.name)


def test_varlen_many_heads_sampled():
    """A causal varlen problem with 64 query heads over 8 KV heads, odd and
    even 256-row block counts, and a one-row and a 255-row sequence, checked
    on sampled rows including every sequence's first and last row."""
    p = workloads.varlen(21, [3000, 2500, 2131, 1900, 255, 1], [3000, 2500, 2131, 1900, 255, 1], 64, 8, 128,
                         "bf16", True)
    _sampled(p, 6, 104)
