"""Pins for the fp64 oracle: checks against what the definition and the pages fix.

None of these compare the oracle with a copy of itself.  Each ``check_*``
helper takes the loaded library so the mutant test at the bottom can run the
same pins against oracle builds with one planted mistake and confirm that
every mistake is caught by at least one pin.
"""
import json
import math
import os
import random

import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import brute
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _lib():
    return oracle.load()


def _packed(seed, lens_q, lens_k, hq, hkv, d, dv=None, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    dv = d if dv is None else dv
    q = torch.randn(sum(lens_q), hq, d, generator=g, dtype=torch.float64).to(dtype)
    k = torch.randn(sum(lens_k), hkv, d, generator=g, dtype=torch.float64).to(dtype)
    v = torch.randn(sum(lens_k), hkv, dv, generator=g, dtype=torch.float64).to(dtype)
    return q, k, v, workloads._cu(lens_q), workloads._cu(lens_k)


# ---------------------------------------------------------------------------
# pins, each usable against a mutant build
# ---------------------------------------------------------------------------

def check_bruteforce(lib):
    """Tiny shapes against the independent pure-Python fsum enumeration."""
    rng = random.Random(7)
    for case in range(24):
        hkv = rng.choice([1, 2])
        hq = hkv * rng.choice([1, 2])
        d = rng.choice([1, 3, 8])
        nseq = rng.choice([1, 2, 3])
        lens_q = [rng.randint(0 if nseq > 1 else 1, 9) for _ in range(nseq)]
        lens_k = [rng.randint(1, 9) for _ in range(nseq)]
        causal = bool(case % 2)
        scale = rng.choice([0.3, 1.0, d ** -0.5])
        q, k, v, cq, ck = _packed(100 + case, lens_q, lens_k, hq, hkv, d)
        o, lse = oracle.attention(q, k, v, cq, ck, scale, causal, lib=lib)
        bo, bl = brute.attention_packed(q.tolist(), k.tolist(), v.tolist(), cq.tolist(), ck.tolist(), scale, causal)
        bo, bl = torch.tensor(bo, dtype=torch.float64).reshape(o.shape), torch.tensor(bl, dtype=torch.float64)
        assert torch.allclose(o, bo, rtol=0, atol=1e-13), (case, (o - bo).abs().max())
        fin = torch.isfinite(bl)
        assert torch.equal(fin, torch.isfinite(lse)), case
        assert torch.allclose(lse[fin], bl[fin], rtol=0, atol=1e-12), case


def check_closed_form(lib):
    spec = json.load(open(os.path.join(GOLD, "closed_form.json")))
    e = math.e
    expect = {
        "two_keys": (lambda p1: [1 + 2 * p1, 2 + 2 * p1])(1 / (e ** 0.5 + 1)),
        "three_keys_equal_and_distinct": [(2 * e + 10 * e ** -2) / (2 * e + e ** -2)] * 2,
    }
    expect_lse = {"two_keys": math.log(e ** 0.5 + 1), "three_keys_equal_and_distinct": math.log(2 * e + e ** -2)}
    for c in spec["cases"]:
        q = torch.tensor(c["q"], dtype=torch.float64)[:, None, :]
        k = torch.tensor(c["k"], dtype=torch.float64)[:, None, :]
        v = torch.tensor(c["v"], dtype=torch.float64)[:, None, :]
        o, lse = oracle.attention(q, k, v, [0, 1], [0, k.shape[0]], c["scale"], False, lib=lib)
        assert torch.allclose(o[0, 0], torch.tensor(expect[c["name"]], dtype=torch.float64), rtol=0, atol=1e-14), c["name"]
        assert abs(float(lse[0, 0]) - expect_lse[c["name"]]) < 1e-14, c["name"]


def check_masked_key_leak(lib):
    spec = json.load(open(os.path.join(GOLD, "masked_key_leak.json")))
    q = torch.tensor(spec["q"], dtype=torch.float64)[:, None, :]
    k = torch.tensor(spec["k"], dtype=torch.float64)[:, None, :]
    v = torch.tensor(spec["v"], dtype=torch.float64)[:, None, :]
    o, lse = oracle.attention(q, k, v, [0, 2], [0, 2], spec["scale"], spec["causal"], lib=lib)
    assert torch.isfinite(o).all()
    assert o[0, 0].abs().max() < spec["page_bound_abs"]
    assert torch.equal(o[0, 0], torch.tensor(spec["expect_row0_o"], dtype=torch.float64))
    assert abs(float(lse[0, 0]) - spec["scale"] * (200 * -100)) < 1e-9


def check_probabilities_sum_to_one(lib):
    q, k, v, cq, ck = _packed(11, [5, 17, 1], [9, 17, 30], 4, 2, 16)
    for causal in (False, True):
        _, lse, ps = oracle.attention(q, k, v, cq, ck, 0.25, causal, lib=lib, return_psum=True)
        fin = torch.isfinite(lse)
        assert torch.allclose(ps[fin], torch.ones_like(ps[fin]), rtol=0, atol=1e-12)


def check_constant_v(lib):
    q, k, v, cq, ck = _packed(12, [7, 33], [40, 33], 2, 1, 8)
    c = torch.linspace(-3, 5, 8, dtype=torch.float64)
    v = c.expand(v.shape[0], v.shape[1], 8).contiguous()
    for causal in (False, True):
        o, _ = oracle.attention(q, k, v, cq, ck, 0.4, causal, lib=lib)
        assert torch.allclose(o, c.expand_as(o), rtol=0, atol=1e-13)


def check_single_visible_key(lib):
    q, k, v, cq, ck = _packed(13, [6], [1], 2, 2, 8)
    o, lse = oracle.attention(q, k, v, cq, ck, 0.7, False, lib=lib)
    for h in range(2):
        assert torch.equal(o[:, h], v[0, h].expand(6, 8))
        s = 0.7 * (q[:, h] * k[0, h]).sum(-1)
        assert torch.allclose(lse[:, h], s, rtol=0, atol=1e-12)


def check_causal_rows(lib):
    """Causal row 0 is v_0; the last causal row equals the non-causal last row
    (oxillama-runtime 0.1.0 flash_attention.rs, test_flash_attention_causal_mask);
    the middle row differs."""
    q, k, v, cq, ck = _packed(14, [8], [8], 1, 1, 4)
    oc, lc = oracle.attention(q, k, v, cq, ck, 0.5, True, lib=lib)
    of, lf = oracle.attention(q, k, v, cq, ck, 0.5, False, lib=lib)
    assert torch.equal(oc[0, 0], v[0, 0])
    assert torch.allclose(oc[7], of[7], rtol=0, atol=1e-14) and torch.allclose(lc[7], lf[7], rtol=0, atol=1e-14)
    assert (oc[4] - of[4]).abs().max() > 1e-4


def check_zero_q_position_code(lib):
    """q = 0 makes every visible score 0: O is the mean of the visible v and
    LSE = ln |V(i)|.  With v_j = (j, j^2) this fixes each row's visible count
    and first key exactly -- the cu_seqlens and mask indexing pin."""
    lens_q, lens_k = [3, 9, 1, 5], [7, 9, 4, 2]
    cq, ck = workloads._cu(lens_q), workloads._cu(lens_k)
    hq, hkv = 4, 2
    q = torch.zeros(sum(lens_q), hq, 4, dtype=torch.float64)
    k = torch.randn(sum(lens_k), hkv, 4, dtype=torch.float64, generator=torch.Generator().manual_seed(3))
    v = torch.zeros(sum(lens_k), hkv, 2, dtype=torch.float64)
    for b in range(4):
        for j in range(lens_k[b]):
            v[ck[b] + j, :, 0] = j
            v[ck[b] + j, :, 1] = j * j
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, cq, ck, 1.0, causal, lib=lib)
        for b in range(4):
            sq, sk = lens_q[b], lens_k[b]
            for i in range(sq):
                vis = [j for j in range(sk) if (not causal) or j <= i + sk - sq]
                t = cq[b] + i
                if not vis:
                    assert torch.all(o[t] == 0) and torch.all(lse[t] == -math.inf)
                    continue
                n = len(vis)
                exp = torch.tensor([sum(vis) / n, sum(j * j for j in vis) / n], dtype=torch.float64)
                assert torch.allclose(o[t], exp.expand(hq, 2), rtol=0, atol=1e-12), (causal, b, i)
                assert torch.allclose(lse[t], torch.full((hq,), math.log(n), dtype=torch.float64), rtol=0, atol=1e-13)


def check_key_shift(lib):
    """k_j -> k_j + u shifts every score of row i by scale*q_i.u: O is
    unchanged and LSE moves by exactly that amount."""
    q, k, v, cq, ck = _packed(15, [9, 4], [9, 11], 2, 2, 8)
    u = torch.randn(8, dtype=torch.float64, generator=torch.Generator().manual_seed(9))
    for causal in (False, True):
        o0, l0 = oracle.attention(q, k, v, cq, ck, 0.3, causal, lib=lib)
        o1, l1 = oracle.attention(q, k + u, v, cq, ck, 0.3, causal, lib=lib)
        assert torch.allclose(o0, o1, rtol=0, atol=1e-12)
        assert torch.allclose(l1 - l0, 0.3 * (q * u).sum(-1), rtol=0, atol=1e-12)


def check_affine_v(lib):
    q, k, v, cq, ck = _packed(16, [6, 10], [12, 10], 2, 1, 8)
    for causal in (False, True):
        o0, _ = oracle.attention(q, k, v, cq, ck, 0.3, causal, lib=lib)
        o1, _ = oracle.attention(q, k, 2.5 * v - 1.25, cq, ck, 0.3, causal, lib=lib)
        assert torch.allclose(o1, 2.5 * o0 - 1.25, rtol=0, atol=1e-12)


def check_permutation(lib):
    q, k, v, cq, ck = _packed(17, [5], [13], 2, 2, 8)
    perm = torch.randperm(13, generator=torch.Generator().manual_seed(1))
    o0, l0 = oracle.attention(q, k, v, cq, ck, 0.3, False, lib=lib)
    o1, l1 = oracle.attention(q, k[perm].contiguous(), v[perm].contiguous(), cq, ck, 0.3, False, lib=lib)
    assert torch.allclose(o0, o1, rtol=0, atol=1e-13) and torch.allclose(l0, l1, rtol=0, atol=1e-13)


def check_torch_sdpa(lib):
    """A third opinion on small cases: torch's float64 SDPA on the CPU with
    an explicit bottom-right boolean mask, K/V repeat_interleave'd for GQA."""
    for causal, (sq, sk) in [(False, (7, 13)), (True, (13, 13)), (True, (5, 11))]:
        q, k, v, cq, ck = _packed(18 + sq, [sq], [sk], 4, 2, 16)
        o, lse = oracle.attention(q, k, v, cq, ck, 0.2, causal, lib=lib)
        qt = q.transpose(0, 1)[None]
        kt = k.repeat_interleave(2, dim=1).transpose(0, 1)[None]
        vt = v.repeat_interleave(2, dim=1).transpose(0, 1)[None]
        mask = None
        if causal:
            mask = torch.arange(sk)[None, :] <= torch.arange(sq)[:, None] + (sk - sq)
        ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.2)[0].transpose(0, 1)
        assert torch.allclose(o, ref, rtol=0, atol=1e-12)
        s = 0.2 * qt @ kt.transpose(-1, -2)
        if mask is not None:
            s = s.masked_fill(~mask, -math.inf)
        assert torch.allclose(lse, torch.logsumexp(s, -1)[0].transpose(0, 1), rtol=0, atol=1e-12)


def check_gqa_and_varlen_structure(lib):
    """GQA == MHA with repeat_interleave'd K/V; packed varlen == per-sequence
    calls (lattice-inference 0.7.1 standard.rs, packed-vs-per-sequence tests)."""
    lens = [5, 1, 12]
    q, k, v, cq, ck = _packed(19, lens, lens, 8, 2, 8)
    o, lse = oracle.attention(q, k, v, cq, ck, 0.3, True, lib=lib)
    o2, l2 = oracle.attention(q, k.repeat_interleave(4, 1).contiguous(), v.repeat_interleave(4, 1).contiguous(),
                              cq, ck, 0.3, True, lib=lib)
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    for b in range(3):
        a, e = int(cq[b]), int(cq[b + 1])
        ob, lb = oracle.attention(q[a:e].contiguous(), k[a:e].contiguous(), v[a:e].contiguous(), [0, e - a], [0, e - a],
                                  0.3, True, lib=lib)
        assert torch.equal(ob, o[a:e]) and torch.equal(lb, lse[a:e])


def check_stability_x50(lib):
    """q, k scaled by 50 (oxillama-runtime flash_attention.rs,
    test_flash_attention_numerical_stability): the result stays finite and
    matches the brute-force enumeration."""
    q, k, v, cq, ck = _packed(20, [16], [16], 1, 1, 8)
    q, k = 50 * q, 50 * k
    o, lse = oracle.attention(q, k, v, cq, ck, 8 ** -0.5, True, lib=lib)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    bo, bl = brute.attention_packed(q.tolist(), k.tolist(), v.tolist(), cq.tolist(), ck.tolist(), 8 ** -0.5, True)
    assert torch.allclose(o, torch.tensor(bo, dtype=torch.float64), rtol=0, atol=1e-12)


def check_mla_views(lib):
    """MLA decode: k = kv[:, :576] and v = kv[:, :512] of one shared head
    (kernelbot-amd-mixed-mla 588924, _bmm_attention), against a float64
    torch.bmm restatement of that materialised path."""
    p = workloads.mla_decode(5, batch=2, q_len=3, kv_len=37, heads=4, dqk=40, dv=32, dtype="bf16")
    o, lse = oracle.problem(p, lib=lib)
    qb = p.q.double().view(2, 3 * 4, 40)
    kvb = p.kv.double().view(2, 37, 40)
    s = torch.bmm(qb, kvb.transpose(1, 2)) * p.scale
    ref = torch.bmm(torch.softmax(s, -1), kvb[:, :, :32]).reshape(6, 4, 32)
    assert torch.allclose(o, ref, rtol=0, atol=1e-12)
    assert torch.allclose(lse, torch.logsumexp(s, -1).reshape(6, 4), rtol=0, atol=1e-12)


PINS = [check_bruteforce, check_closed_form, check_masked_key_leak, check_probabilities_sum_to_one,
        check_constant_v, check_single_visible_key, check_causal_rows, check_zero_q_position_code,
        check_key_shift, check_affine_v, check_permutation, check_torch_sdpa,
        check_gqa_and_varlen_structure, check_stability_x50, check_mla_views]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(_lib())


def test_storage_dtypes_upcast_exactly():
    """bf16 / f16 / f32 inputs are read as their exact values: every f16 bit
    pattern (subnormals, +-0, +-inf) and a spread of bf16 ones."""
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    for dt in (torch.float16, torch.bfloat16):
        vals = bits.view(dt)
        finite = vals[torch.isfinite(vals.float())]
        n = finite.numel() - finite.numel() % 64
        v = finite[:n].reshape(n // 64, 1, 64)
        # one key, so O == v exactly; q = 0 keeps the score finite
        q = torch.zeros(1, 1, 64, dtype=dt)
        for r in range(0, v.shape[0], 97):
            o, _ = oracle.attention(q, torch.zeros(1, 1, 64, dtype=dt), v[r:r + 1].contiguous(), [0, 1], [0, 1],
                                    1.0, False)
            assert torch.equal(o[0, 0], v[r, 0].double())
    x = torch.randn(3, 1, 8, dtype=torch.float32)
    o32, _ = oracle.attention(x, x, x, [0, 3], [0, 3], 0.5, True)
    o64, _ = oracle.attention(x.double(), x.double(), x.double(), [0, 3], [0, 3], 0.5, True)
    assert torch.equal(o32, o64)


def test_row_subset_matches_full():
    p = workloads.varlen(21, [33, 2, 64], [40, 2, 64], 4, 2, 16, "bf16", True)
    o, lse = oracle.problem(p)
    pairs = workloads.sample_rows(p, 5, 0)
    os_, ls = oracle.problem(p, pairs=pairs)
    assert torch.equal(os_, o[pairs[:, 0], pairs[:, 1]]) and torch.equal(ls, lse[pairs[:, 0], pairs[:, 1]])


def test_workload_recipe_lengths():
    """The varlen workload's lengths come from torch.randint(128, 4097, (16,))
    on a CPU generator seeded 2."""
    _, lens = workloads.varlen_lengths()
    assert len(lens) == 16 and all(128 <= n <= 4096 for n in lens)
    assert lens == workloads.varlen_lengths()[1]


MUTANTS = {1: "scale dropped", 2: "h % Hkv head map", 3: "diagonal masked", 4: "top-left causal",
           5: "reversed k operand", 6: "score sign flipped", 7: "normalisation dropped",
           8: "wrong sequence lookup", 9: "k used as v", 10: "log dropped from LSE"}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=[MUTANTS[m] for m in sorted(MUTANTS)])
def test_pins_catch_planted_mistake(mutant, tmp_path):
    """Each plausible mistake, planted in a separate oracle build on the CPU,
    fails at least one pin."""
    lib = oracle.load(oracle.build(str(tmp_path / f"liboracle_m{mutant}.so"), mutant=mutant))
    caught = []
    for pin in PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError):
            caught.append(pin.__name__)
    assert caught, f"mutant {mutant} ({MUTANTS[mutant]}) passed every pin"


# ---------------------------------------------------------------------------
# E4M3 codes (oracle/e4m3.py) and the oracle over an fp8 latent cache
# ---------------------------------------------------------------------------

def test_e4m3_closed_forms():
    """Values the E4M3 definition fixes by itself."""
    from oracle import e4m3
    assert e4m3.value(0x00) == 0.0 and math.copysign(1.0, e4m3.value(0x00)) == 1.0
    assert e4m3.value(0x80) == 0.0 and math.copysign(1.0, e4m3.value(0x80)) == -1.0
    assert e4m3.value(0x38) == 1.0           # exponent field = bias, mantissa 0
    assert e4m3.value(0xB8) == -1.0
    assert e4m3.value(0x3C) == 1.5
    assert e4m3.value(0x7E) == 448.0         # largest finite value
    assert e4m3.value(0x08) == 2.0 ** -6     # smallest normal
    assert e4m3.value(0x01) == 2.0 ** -9     # smallest subnormal
    assert e4m3.value(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert math.isnan(e4m3.value(0x7F)) and math.isnan(e4m3.value(0xFF))


def test_e4m3_matches_torch_float8_for_every_code():
    """torch's own float8_e4m3fn -> float64 conversion, written independently
    of oracle/e4m3.py, agrees on all 256 codes (signs of zero included)."""
    from oracle import e4m3
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64)
    got = e4m3.decode(codes)
    nan = torch.isnan(ref)
    assert torch.equal(nan, torch.isnan(got)) and int(nan.sum()) == 2
    assert torch.equal(got[~nan], ref[~nan])
    assert torch.equal(torch.signbit(got[~nan]), torch.signbit(ref[~nan]))


def test_e4m3_order_and_sign():
    from oracle import e4m3
    vals = [e4m3.value(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    assert all(e4m3.value(c | 0x80) == -e4m3.value(c) for c in range(0x7F))


def test_fp8_mla_oracle_matches_brute_force():
    """oracle.problem over an E4M3 cache equals the pure-Python restatement
    given torch's own dequantisation (torch's float8 cast times the scale,
    value = the first 512 columns)."""
    p = workloads.mla_decode_fp8(31, batch=2, q_len=2, kv_len=0, heads=2, lens_kv=[3, 5], causal=True)
    o, lse = oracle.problem(p)
    kv = p.kv.view(torch.float8_e4m3fn).to(torch.float64) * p.kv_scale
    bo, bl = brute.attention_packed(p.q.double().tolist(), kv.view(-1, 1, 576).tolist(),
                                    kv[:, :512].reshape(-1, 1, 512).tolist(), p.cu_q.tolist(), p.cu_k.tolist(),
                                    p.scale, p.causal)
    assert torch.allclose(o, torch.tensor(bo, dtype=torch.float64), rtol=0, atol=1e-12)
    assert torch.allclose(lse, torch.tensor(bl, dtype=torch.float64), rtol=0, atol=1e-12)


def test_fp8_workload_codes_are_finite_and_span_the_range():
    p = workloads.mla_decode_fp8(32, batch=2, q_len=4, kv_len=300)
    vals = p.kv.view(torch.float8_e4m3fn).to(torch.float64)
    assert not torch.isnan(vals).any()
    assert vals.abs().max().item() == 448.0
    assert p.kv.dtype == torch.uint8 and tuple(p.kv.shape) == (600, 576)
