"""KV-cache decode (dense and paged caches, append) against the fp64 oracle."""
import pytest
import torch

import oracle
import workloads
from parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import tiled_attention_21_b200 as mx
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mx.load()


def run_case(w, causal=False, num_splits=0):
    import tiled_attention_21_b200 as mx
    dev = torch.device("cuda")
    q = w["q"].to(dev)
    kc, vc = w["k_cache"].to(dev), w["v_cache"].to(dev)
    kn = None if w["k_new"] is None else w["k_new"].to(dev)
    vn = None if w["v_new"] is None else w["v_new"].to(dev)
    sl = w["cache_seqlens"].to(dev)
    bt = None if w["block_table"] is None else w["block_table"].to(dev)
    kc0, vc0 = kc.clone(), vc.clone()
    o, lse = mx.mxfa_attn_decode_kvcache(q, kc, vc, sl, kn, vn, bt, causal=causal, num_splits=num_splits)
    torch.cuda.synchronize()
    p = w["problem"]
    p.causal = causal
    ro, rl = oracle.problem(p)
    B, Sq, Hq, D = q.shape
    compare(o.reshape(B * Sq, Hq, D), lse.reshape(B * Sq, Hq), ro, rl, p.q.dtype, p.name)
    # the append wrote exactly the new rows, and advanced the lengths
    snew = 0 if kn is None else kn.shape[1]
    seq0 = w["cache_seqlens"].tolist()
    assert sl.cpu().tolist() == [L + snew for L in seq0]
    exp_k, exp_v = kc0.cpu(), vc0.cpu()
    for b in range(B):
        for i in range(snew):
            pg, off = w["rows"](b, seq0[b] + i)
            exp_k[pg, off], exp_v[pg, off] = w["k_new"][b, i], w["v_new"][b, i]
    assert torch.equal(kc.cpu(), exp_k) and torch.equal(vc.cpu(), exp_v)
    return o, lse


@pytest.mark.parametrize("page_size", [16, 64, 128, 256])
def test_paged(page_size):
    w = workloads.kvcache(41, batch=4, Sq=1, Snew=0, seqlens=[1, 300, 1024, 777], page_size=page_size)
    run_case(w)


def test_dense_ragged():
    w = workloads.kvcache(42, batch=3, Sq=1, Snew=0, seqlens=[5, 200, 999], cache_len=1100)
    run_case(w)


@pytest.mark.parametrize("page_size", [None, 32, 128])
def test_append_causal(page_size):
    # Sq = Snew new tokens attend to the cache and to each other causally
    w = workloads.kvcache(43, batch=3, Sq=4, Snew=4, seqlens=[0, 129, 640], page_size=page_size, cache_len=700,
                          causal=True)
    run_case(w, causal=True)


def test_append_single_token_gqa16_d64():
    w = workloads.kvcache(44, batch=2, Sq=1, Snew=1, seqlens=[63, 64], hq=16, hkv=1, d=64, dtype="f16",
                          page_size=64)
    run_case(w)


def test_head_groups_sq16():
    # 16 queries x 8 heads per KV head = 128 rows: two head groups per KV head
    w = workloads.kvcache(48, batch=2, Sq=16, Snew=16, seqlens=[100, 300], page_size=64, causal=True)
    run_case(w, causal=True)


def test_split_invariance():
    w = workloads.kvcache(45, batch=2, Sq=1, Snew=0, seqlens=[3000, 4096], page_size=128)
    o1, l1 = run_case(w, num_splits=1)
    o8, l8 = run_case(w, num_splits=8)
    assert (o1.float() - o8.float()).abs().max() <= 4e-3
    assert (l1 - l8).abs().max() <= 1e-4


def test_append_past_capacity_is_reported():
    import tiled_attention_21_b200 as mx
    dev = torch.device("cuda")
    w = workloads.kvcache(46, batch=1, Sq=1, Snew=0, seqlens=[16], page_size=16)
    kc, vc = w["k_cache"].to(dev), w["v_cache"].to(dev)
    kc0 = kc.clone()
    table = w["block_table"].to(dev)  # one page of 16 positions
    sl = torch.tensor([16], dtype=torch.int32, device=dev)
    kn = torch.ones((1, 1, 4, 128), dtype=kc.dtype, device=dev)
    ws = mx.workspace(1 << 20, dev)
    mx.mxfa_attn_decode_kvcache(w["q"].to(dev), kc, vc, sl, kn, kn.clone(), table, ws=ws)
    st, site = mx.read_device_status(ws)
    assert st == mx.MXFA_ERR_INVALID_ARG and site == 0x501
    assert torch.equal(kc, kc0)  # nothing written


def test_dense_length_past_capacity_is_reported():
    """A dense cache entry holds page_size (= the cache length) keys; a
    cache_seqlens value beyond it is cut there and reported (site 0x402), so
    no key of the next entry is read."""
    import tiled_attention_21_b200 as mx
    dev = torch.device("cuda")
    w = workloads.kvcache(47, batch=2, Sq=1, Snew=0, seqlens=[64, 30], cache_len=64)
    kc, vc = w["k_cache"].to(dev), w["v_cache"].to(dev)
    sl = torch.tensor([100, 30], dtype=torch.int32, device=dev)
    ws = mx.workspace(1 << 20, dev)
    o, lse = mx.mxfa_attn_decode_kvcache(w["q"].to(dev), kc, vc, sl, ws=ws)
    st, site = mx.read_device_status(ws)
    assert (st, site) == (mx.MXFA_ERR_INVALID_ARG, 0x402)
    p = w["problem"]  # the 64 cached keys of entry 0, 30 of entry 1
    ro, rl = oracle.problem(p)
    B, Sq, Hq, D = w["q"].shape
    compare(o.reshape(B * Sq, Hq, D), lse.reshape(B * Sq, Hq), ro, rl, p.q.dtype, "dense past capacity")
