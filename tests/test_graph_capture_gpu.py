"""The entry points enqueue only stream work (kernel launches, including the
cooperative one-launch decode, and a memset), so a call can be captured in a
CUDA graph and replayed.  Each case captures one call, refills the inputs in
place with new values, replays, and compares with a direct call on the same
inputs."""
import pytest
import torch

import workloads
from runners import run, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import tiled_attention_21_b200 as mx
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mx.load()


def _replay_matches(p_a, p_b, entry):
    """Capture `entry` on p_a's inputs, refill them with p_b's, replay, and
    compare with a direct call on p_b."""
    import tiled_attention_21_b200 as mx
    d = to_dev(p_a)
    o = torch.empty(p_a.total_q, p_a.hq, p_a.dv, dtype=p_a.q.dtype, device="cuda")
    lse = torch.empty(p_a.total_q, p_a.hq, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run(p_a, d, entry, out=o, lse=lse, stream=s)  # warm-up: kernel attributes set outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(p_a, d, entry, out=o, lse=lse, stream=s)
    src = to_dev(p_b)
    for key in ("q", "k", "v", "kv"):
        if key in d and key in src:
            d[key].copy_(src[key])
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert mx.read_device_status()[0] == 0
    o_ref, l_ref = run(p_b, src, entry)
    torch.cuda.synchronize()
    assert torch.equal(o.float(), o_ref.float())
    assert torch.equal(lse, l_ref)


def test_graph_mla_decode_single_launch():
    # small problem: the one-launch cooperative decode
    a = workloads.mla_decode(51, batch=4, q_len=4, kv_len=1024)
    b = workloads.mla_decode(52, batch=4, q_len=4, kv_len=1024)
    _replay_matches(a, b, "decode")


def test_graph_mla_decode_three_kernels():
    # larger problem: schedule, decode and combine kernels
    a = workloads.mla_decode(53, batch=64, q_len=4, kv_len=2048)
    b = workloads.mla_decode(54, batch=64, q_len=4, kv_len=2048)
    _replay_matches(a, b, "decode")


def test_graph_gqa_decode():
    a = workloads.gqa_decode(55, batch=4, q_len=1, kv_len=3000)
    b = workloads.gqa_decode(56, batch=4, q_len=1, kv_len=3000)
    _replay_matches(a, b, "decode")


def test_graph_varlen_prefill():
    lens = [300, 1000, 77]
    a = workloads.varlen(57, lens, lens, 8, 2, 128, "bf16", True)
    b = workloads.varlen(58, lens, lens, 8, 2, 128, "bf16", True)
    _replay_matches(a, b, "varlen")


def test_graph_mla_decode_fp8kv():
    a = workloads.mla_decode_fp8(59, batch=4, q_len=4, kv_len=1024)
    b = workloads.mla_decode_fp8(60, batch=4, q_len=4, kv_len=1024)
    b.kv_scale = a.kv_scale  # the scale is a call argument, captured with the graph
    _replay_matches(a, b, "decode")


def test_graph_mla_decode_head_groups():
    # 8 queries x 16 heads: two head groups, three kernels (more sequences than one launch takes)
    a = workloads.mla_decode(61, batch=96, q_len=8, kv_len=1500)
    b = workloads.mla_decode(62, batch=96, q_len=8, kv_len=1500)
    _replay_matches(a, b, "decode")
