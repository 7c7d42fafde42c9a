"""A bounded device wait that runs out (the failure-detection path).

Every spin in the kernels is bounded by a budget carried in the launch
parameters (2 s by default).  This test shortens the budget to 1 ms through
the library's testing hook and makes one wait unsatisfiable from the host:
the one-launch MLA decode merges the pieces of a split sequence after each
piece has counted itself in a per-sequence counter of the workspace, and the
hook keeps the counters the test prepared (hugely negative) instead of
zeroing them, so the count never reaches the number of pieces.  The call
must return, report MXFA_ERR_TIMEOUT at the merge's wait site, and leave the
GPU usable: the next normal call on the same workspace matches the oracle.
No fault, trap or endless loop is involved (oxillama-runtime 0.1.0
flash_attention.rs returns its errors as values; so does this library).
"""
import pytest
import torch

import oracle
import workloads
from parity import compare
from runners import to_dev

pytestmark = pytest.mark.gpu

SITE_MERGE = 0x309


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import tiled_attention_21_b200 as mx
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mx.load()


def test_merge_wait_runs_out_and_the_next_call_is_clean():
    import tiled_attention_21_b200 as mx
    lib = mx.load()
    # batch 2 x 16 KV tiles: the one-launch schedule, each sequence in 8 pieces
    p = workloads.mla_decode(61, batch=2, q_len=4, kv_len=1024)
    d = to_dev(p)
    need = lib.mxfa_attn_decode_splitkv_workspace_size(p.batch, 4, p.hq, 1, p.dv, 1024, 0, 2)
    ws = torch.full((need + 512,), 0x80, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    ws[off:off + 256].zero_()  # the status header starts clear; the counters read 0x80808080 < 0

    def call():
        return mx.mxfa_attn_decode_splitkv(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"], 4, 1024,
                                           softmax_scale=p.scale, ws=ws)

    lib.mxfa_test_hooks(1_000_000, 1)  # 1 ms budget, keep the prepared counters
    try:
        call()
        st, site = mx.read_device_status(ws)
    finally:
        lib.mxfa_test_hooks(0, 0)
    assert (st, site) == (mx.MXFA_ERR_TIMEOUT, SITE_MERGE)
    o, l = call()
    torch.cuda.synchronize()
    assert mx.read_device_status(ws)[0] == mx.MXFA_OK
    ro, rl = oracle.problem(p)
    compare(o, l, ro, rl, p.q.dtype, "after a timed-out call")
