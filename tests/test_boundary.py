"""The C-ABI library: it loads without a GPU, exports every function the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxfa.h")


@pytest.fixture(scope="module")
def lib():
    from tiled_attention_21_b200 import build_ext
    import tiled_attention_21_b200 as m
    try:
        build_ext.build()
    except RuntimeError as e:  # no nvcc
        if not os.path.exists(m.LIB_PATH):
            pytest.skip(str(e))
    return m.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mxfa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_three_entry_points():
    names = declared_functions()
    for n in ("mxfa_attn_fwd", "mxfa_attn_varlen_fwd", "mxfa_attn_decode_splitkv", "mxfa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from tiled_attention_21_b200 import LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\S+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        getattr(lib, n)


FAKE = 0x100000  # never dereferenced: every call below fails validation first


def fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Sq=8, Sk=8, Hq=2, Hkv=1, D=64, dt=2,
             qr=128, qh=64, kr=64, kh=64, vr=64, vh=64, orr=128, oh=64, scale=float("nan"), causal=0,
             ws=FAKE, wsn=4096)
    a.update(kw)
    return lib.mxfa_attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Sq"], a["Sk"], a["Hq"], a["Hkv"],
                             a["D"], a["dt"], a["qr"], a["qh"], a["kr"], a["kh"], a["vr"], a["vh"], a["orr"], a["oh"],
                             a["scale"], a["causal"], a["ws"], a["wsn"], None)


def test_validation_errors(lib):
    import tiled_attention_21_b200 as m
    assert fwd(lib, Hq=3, Hkv=2) == m.MXFA_ERR_INVALID_ARG
    assert b"multiple" in lib.mxfa_last_error()
    assert fwd(lib, D=96) == m.MXFA_ERR_UNSUPPORTED
    assert fwd(lib, dt=7) == m.MXFA_ERR_INVALID_ARG
    assert fwd(lib, q=None) == m.MXFA_ERR_INVALID_ARG
    assert fwd(lib, q=FAKE + 8) == m.MXFA_ERR_INVALID_ARG
    assert fwd(lib, qr=100) == m.MXFA_ERR_INVALID_ARG  # 200 bytes: not a multiple of 16
    assert fwd(lib, ws=None) == m.MXFA_ERR_WORKSPACE
    assert fwd(lib, ws=FAKE + 16) == m.MXFA_ERR_WORKSPACE
    assert fwd(lib, wsn=16) == m.MXFA_ERR_WORKSPACE
    assert fwd(lib, B=-1) == m.MXFA_ERR_INVALID_ARG
    assert fwd(lib, scale=float("inf")) == m.MXFA_ERR_INVALID_ARG
    # empty problems are a no-op and succeed without touching the device
    assert fwd(lib, B=0) == m.MXFA_OK
    assert fwd(lib, Sq=0) == m.MXFA_OK


def test_varlen_and_decode_validation(lib):
    import tiled_attention_21_b200 as m
    r = lib.mxfa_attn_varlen_fwd(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 2, 10, 10, 8, 8, 4, 2, 128, 2,
                                 float("nan"), 1, FAKE, 1 << 20, None)
    assert r == m.MXFA_ERR_INVALID_ARG  # cu_seqlens_q NULL
    r = lib.mxfa_attn_varlen_fwd(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 10, 10, 11, 8, 4, 2, 128, 2,
                                 float("nan"), 1, FAKE, 1 << 20, None)
    assert r == m.MXFA_ERR_INVALID_ARG  # max_seqlen_q > total_q
    r = lib.mxfa_attn_decode_splitkv(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 8, 64, 4, 32, 16, 1, 576, 256,
                                     576, 576, 2, float("nan"), 0, 0, FAKE, 1 << 20, None)
    assert r == m.MXFA_ERR_UNSUPPORTED  # (576, 256)
    r = lib.mxfa_attn_decode_splitkv(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 8, 64, 4, 32, 16, 1, 576, 512,
                                     500, 576, 2, float("nan"), 0, 0, FAKE, 1 << 20, None)
    assert r == m.MXFA_ERR_INVALID_ARG  # k row stride shorter than a row
    r = lib.mxfa_attn_decode_splitkv(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 8, 64, 4, 32, 16, 1, 576, 512,
                                     576, 576, 2, float("nan"), 0, -1, FAKE, 1 << 20, None)
    assert r == m.MXFA_ERR_INVALID_ARG  # negative split count


def test_fp8_decode_validation(lib):
    import tiled_attention_21_b200 as m

    def c(**kw):
        a = dict(q=FAKE, kv=FAKE, ks=0.25, o=FAKE, lse=None, qo=FAKE, kvi=FAKE, B=2, tq=8, tkv=64, mq=4, mkv=32,
                 Hq=16, rs=576, scale=float("nan"), causal=0, splits=0, ws=FAKE, wn=1 << 20)
        a.update(kw)
        return lib.mxfa_attn_decode_mla_fp8kv(a["q"], a["kv"], a["ks"], a["o"], a["lse"], a["qo"], a["kvi"], a["B"],
                                              a["tq"], a["tkv"], a["mq"], a["mkv"], a["Hq"], a["rs"], a["scale"],
                                              a["causal"], a["splits"], a["ws"], a["wn"], None)

    assert c(mq=65, tq=130) == m.MXFA_ERR_UNSUPPORTED      # more than 64 queries per sequence
    assert c(ks=float("inf")) == m.MXFA_ERR_INVALID_ARG     # scale not finite
    assert c(ks=float("nan")) == m.MXFA_ERR_INVALID_ARG
    assert c(rs=560) == m.MXFA_ERR_INVALID_ARG              # row shorter than 576 codes
    assert c(rs=584) == m.MXFA_ERR_INVALID_ARG              # not a multiple of 16 bytes
    assert c(kv=None) == m.MXFA_ERR_INVALID_ARG
    assert c(kvi=None) == m.MXFA_ERR_INVALID_ARG
    assert c(splits=-1) == m.MXFA_ERR_INVALID_ARG
    assert c(wn=16) == m.MXFA_ERR_WORKSPACE
    assert c(B=0) == m.MXFA_OK                              # nothing to do
    need = lib.mxfa_attn_decode_mla_fp8kv_workspace_size(128, 4, 16, 8192, 0)
    assert need > 256 and need == lib.mxfa_attn_decode_splitkv_workspace_size(128, 4, 16, 1, 512, 8192, 0, 2)
    # 8 x 16 query rows: two head groups, each a decode sequence of its own
    need8 = lib.mxfa_attn_decode_mla_fp8kv_workspace_size(128, 8, 16, 8192, 0)
    assert need8 > need and need8 == lib.mxfa_attn_decode_splitkv_workspace_size(128, 8, 16, 1, 512, 8192, 0, 2)
    assert lib.mxfa_attn_decode_mla_fp8kv_workspace_size(128, 65, 16, 8192, 0) == 256


def test_workspace_sizes(lib):
    assert lib.mxfa_attn_fwd_workspace_size(4, 2048, 2048, 16, 16, 128, 2) >= 256
    small = lib.mxfa_attn_varlen_fwd_workspace_size(2, 128, 128, 8, 128, 2)
    big = lib.mxfa_attn_varlen_fwd_workspace_size(64, 32768, 32768, 8, 128, 2)
    assert 256 < small < big
    assert lib.mxfa_attn_varlen_fwd_workspace_size(2, 128, 128, 8, 128, 0) == 256  # fp32 path needs no schedule
    mla = lib.mxfa_attn_decode_splitkv_workspace_size(128, 4, 16, 1, 512, 8192, 0, 2)
    gqa = lib.mxfa_attn_decode_splitkv_workspace_size(64, 1, 32, 4, 128, 8192, 0, 2)
    assert mla > 256 and gqa > 256
    # the grouped-query schedule covers batch * Hkv sequences
    assert lib.mxfa_attn_decode_splitkv_workspace_size(64, 1, 32, 8, 128, 8192, 0, 2) > gqa
    assert lib.mxfa_attn_decode_splitkv_workspace_size(64, 1, 32, 4, 128, 8192, 0, 0) == 256  # fp32


def test_product_path_does_not_touch_the_oracle():
    """The package never imports, loads or builds anything under oracle/."""
    pkg = os.path.join(ROOT, "tiled_attention_21_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f


def test_kvcache_validation(lib):
    import tiled_attention_21_b200 as m
    call = lib.mxfa_attn_decode_kvcache

    def c(**kw):
        a = dict(q=FAKE, kc=FAKE, vc=FAKE, kn=None, vn=None, sl=FAKE, bt=FAKE, B=2, Sq=1, Snew=0, Hq=32, Hkv=4, D=128,
                 pages=8, page=64, blocks=4, max_len=256, dt=2, scale=float("nan"), causal=0, splits=0, o=FAKE,
                 lse=None, ws=FAKE, wn=1 << 20)
        a.update(kw)
        return call(a["q"], a["kc"], a["vc"], a["kn"], a["vn"], a["sl"], a["bt"], a["B"], a["Sq"], a["Snew"],
                    a["Hq"], a["Hkv"], a["D"], a["pages"], a["page"], a["blocks"], a["max_len"], a["dt"], a["scale"],
                    a["causal"], a["splits"], a["o"], a["lse"], a["ws"], a["wn"], None)

    assert c(D=96) == m.MXFA_ERR_UNSUPPORTED                 # head dim
    assert c(dt=0) == m.MXFA_ERR_UNSUPPORTED                 # fp32
    assert c(Sq=65) == m.MXFA_ERR_UNSUPPORTED                # more than 64 queries per sequence
    assert c(page=48) == m.MXFA_ERR_UNSUPPORTED              # page size
    assert c(Hq=30) == m.MXFA_ERR_INVALID_ARG                # Hq not a multiple of Hkv
    assert c(Snew=2) == m.MXFA_ERR_INVALID_ARG               # appended rows without k_new / v_new
    assert c(sl=None) == m.MXFA_ERR_INVALID_ARG              # cache_seqlens missing
    assert c(bt=None, pages=3) == m.MXFA_ERR_INVALID_ARG     # dense cache: one page per batch entry
    assert c(blocks=0) == m.MXFA_ERR_INVALID_ARG             # empty block table
    assert c(wn=16) == m.MXFA_ERR_WORKSPACE                  # workspace too small
    assert c(B=0) == m.MXFA_OK                               # nothing to do
    need = lib.mxfa_attn_decode_kvcache_workspace_size(64, 1, 32, 4, 128, 8192, 0, 2)
    assert need > 256 and need == lib.mxfa_attn_decode_splitkv_workspace_size(64, 1, 32, 4, 128, 8192, 0, 2)


def test_fp8_binding_rejects_bad_tensors(lib):
    """The binding checks dtypes and layouts before any device work."""
    import torch
    import tiled_attention_21_b200 as m
    q = torch.zeros(8, 16, 576, dtype=torch.bfloat16)
    kv = torch.zeros(64, 576, dtype=torch.uint8)
    cu = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError):  # q must be bf16
        m.mxfa_attn_decode_mla_fp8kv(q.float(), kv, 1.0, cu, cu, 4, 32)
    with pytest.raises(ValueError):  # q must be contiguous
        m.mxfa_attn_decode_mla_fp8kv(q.transpose(0, 1), kv, 1.0, cu, cu, 4, 32)
    with pytest.raises(ValueError):  # codes are bytes
        m.mxfa_attn_decode_mla_fp8kv(q, kv.to(torch.int16), 1.0, cu, cu, 4, 32)
    with pytest.raises(ValueError):  # [total_kv, 576] with unit stride inside a row
        m.mxfa_attn_decode_mla_fp8kv(q, kv.view(64, 1, 576), 1.0, cu, cu, 4, 32)
    with pytest.raises(ValueError):
        m.mxfa_attn_decode_mla_fp8kv(q, kv.t(), 1.0, cu, cu, 4, 32)
