"""Seeded synthetic inputs for the attention forward workloads.

This module only draws random numbers and lays them out; it holds none of
the attention arithmetic. Both the fp64 oracle (under ``oracle/``) and the
CUDA path consume what it returns, so it is the one module they share.

Recipe (every value i.i.d. N(0, 1) unless stated):
  * a ``torch.Generator('cpu')`` seeded with the workload's seed;
  * ``torch.randn(shape, dtype=float32, generator=g)`` drawn in the order
    q, k, v (MLA decode: q, kv);
  * then a cast to the workload's dtype with round-to-nearest-even.
The shapes follow the pages' own workloads: the flash_attn layouts
``[B, S, H, D]`` / ``[total_tokens, H, D]`` of mxflashattn 1.4.0
(``flash_attn_func``, ``flash_attn_varlen_func``) and the MLA decode inputs
``(q, kv, qo_indptr, kv_indptr)`` of kernelbot-amd-mixed-mla submission
588924 (``custom_kernel``).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass
class Problem:
    """One attention forward problem in packed (varlen) form.

    q: [total_q, Hq, Dqk]; k: [total_k, Hkv, Dqk]; v: [total_k, Hkv, Dv]
    (for MLA decode k and v are views of one kv tensor [total_k, 1, 576]).
    cu_q / cu_k: int32 [batch + 1] cumulative lengths.
    ``batched`` is set when every sequence has the same length, so the
    tensors can also be viewed as [B, S, H, D].
    """

    name: str
    dtype: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    cu_q: torch.Tensor
    cu_k: torch.Tensor
    hq: int
    hkv: int
    dqk: int
    dv: int
    causal: bool
    scale: float
    batched: bool = False
    mla: bool = False
    kv: torch.Tensor | None = None  # MLA: the single [total_k, 576] cache
    kv_scale: float | None = None  # set: kv holds E4M3 codes (uint8), element = kv_scale * code value
    check_rows: torch.Tensor | None = None  # [n, 2] (token, head) pairs the oracle evaluates
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.cu_q.numel() - 1

    @property
    def total_q(self) -> int:
        return int(self.cu_q[-1])

    @property
    def total_k(self) -> int:
        return int(self.cu_k[-1])

    def seqlens_q(self) -> list[int]:
        c = self.cu_q.tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]

    def seqlens_k(self) -> list[int]:
        c = self.cu_k.tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]


def _cu(lengths: list[int]) -> torch.Tensor:
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return torch.tensor(out, dtype=torch.int32)


def _randn(g: torch.Generator, shape, dtype: str) -> torch.Tensor:
    return torch.randn(shape, dtype=torch.float32, generator=g).to(DTYPES[dtype])


def batched(seed: int, B: int, Sq: int, Sk: int, Hq: int, Hkv: int, D: int, dtype: str,
            causal: bool, scale: float | None = None, name: str = "batched",
            Dv: int | None = None) -> Problem:
    """[B, S, H, D] inputs, stored packed as [B*S, H, D]."""
    Dv = D if Dv is None else Dv
    g = torch.Generator("cpu").manual_seed(seed)
    q = _randn(g, (B, Sq, Hq, D), dtype).reshape(B * Sq, Hq, D)
    k = _randn(g, (B, Sk, Hkv, D), dtype).reshape(B * Sk, Hkv, D)
    v = _randn(g, (B, Sk, Hkv, Dv), dtype).reshape(B * Sk, Hkv, Dv)
    return Problem(name, dtype, q, k, v, _cu([Sq] * B), _cu([Sk] * B), Hq, Hkv, D, Dv, causal,
                   D ** -0.5 if scale is None else scale, batched=True,
                   meta={"B": B, "Sq": Sq, "Sk": Sk})


def varlen(seed: int, lens_q: list[int], lens_k: list[int], Hq: int, Hkv: int, D: int, dtype: str,
           causal: bool, scale: float | None = None, name: str = "varlen") -> Problem:
    g = torch.Generator("cpu").manual_seed(seed)
    tq, tk = sum(lens_q), sum(lens_k)
    q = _randn(g, (tq, Hq, D), dtype)
    k = _randn(g, (tk, Hkv, D), dtype)
    v = _randn(g, (tk, Hkv, D), dtype)
    return Problem(name, dtype, q, k, v, _cu(lens_q), _cu(lens_k), Hq, Hkv, D, D, causal,
                   D ** -0.5 if scale is None else scale)


def mla_decode(seed: int, batch: int, q_len: int, kv_len: int, heads: int = 16, dqk: int = 576,
               dv: int = 512, dtype: str = "bf16", name: str = "mla_decode",
               lens_kv: list[int] | None = None) -> Problem:
    """MLA decode: q [batch*q_len, heads, 576]; one shared kv head [total_kv, 576];
    k = kv[:, :576], v = kv[:, :512] (kernelbot-amd-mixed-mla 588924, ``_flash_fused``)."""
    g = torch.Generator("cpu").manual_seed(seed)
    lens_kv = [kv_len] * batch if lens_kv is None else lens_kv
    tk = sum(lens_kv)
    q = _randn(g, (batch * q_len, heads, dqk), dtype)
    kv = _randn(g, (tk, dqk), dtype)
    k = kv.view(tk, 1, dqk)
    v = kv[:, :dv].view(tk, 1, dv)  # a strided view: row stride 576
    return Problem(name, dtype, q, k, v, _cu([q_len] * batch), _cu(lens_kv), heads, 1, dqk, dv,
                   False, dqk ** -0.5, mla=True, kv=kv,
                   meta={"batch": batch, "q_len": q_len, "kv_len": kv_len})


def mla_decode_fp8(seed: int, batch: int, q_len: int, kv_len: int, heads: int = 16,
                   lens_kv: list[int] | None = None, causal: bool = False,
                   name: str = "mla_decode_fp8") -> Problem:
    """MLA decode over an E4M3 latent cache: q [batch*q_len, heads, 576] bf16;
    kv [total_kv, 576] E4M3 codes (uint8) with one fp32 scale.  Recipe: q as
    in ``mla_decode``; the cache is drawn as N(0, 1) fp32 values x (after q,
    from the same generator), the scale is the fp32 value of max|x| / 448 (the
    codes then span the format's range, 448 being its largest finite value),
    and the codes are torch's round-to-nearest-even cast of x / scale, clamped
    to [-448, 448], to float8_e4m3fn."""
    g = torch.Generator("cpu").manual_seed(seed)
    lens_kv = [kv_len] * batch if lens_kv is None else lens_kv
    tk = sum(lens_kv)
    q = _randn(g, (batch * q_len, heads, 576), "bf16")
    x = torch.randn((tk, 576), dtype=torch.float32, generator=g)
    amax = float(x.abs().max()) if tk else 448.0
    scale = float(torch.tensor(amax / 448.0, dtype=torch.float32))
    codes = (x / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return Problem(name, "bf16", q, codes.view(tk, 1, 576), codes[:, :512].view(tk, 1, 512),
                   _cu([q_len] * batch), _cu(lens_kv), heads, 1, 576, 512, causal, 576 ** -0.5, mla=True,
                   kv=codes, kv_scale=scale, meta={"batch": batch, "q_len": q_len, "kv_len": kv_len})


def gqa_decode(seed: int, batch: int, q_len: int, kv_len: int, hq: int = 32, hkv: int = 4, d: int = 128,
               dtype: str = "bf16", causal: bool = False, lens_kv: list[int] | None = None,
               name: str | None = None) -> Problem:
    """Grouped-query decode on a dense KV cache: q [batch*q_len, hq, d], k/v
    [total_kv, hkv, d] (the q_len = 1 decode bench shapes of AstrAI
    attn_decode_split_kv_mma.cuh: Hq = 32, Hk = 4, D = 128)."""
    lens_kv = [kv_len] * batch if lens_kv is None else lens_kv
    return varlen(seed, [q_len] * batch, lens_kv, hq, hkv, d, dtype, causal,
                  name=name or f"gqa_decode_b{batch}_q{q_len}_kv{kv_len}_hq{hq}_hkv{hkv}_d{d}_{dtype}")


# ---------------------------------------------------------------------------
# The five named workloads.
# ---------------------------------------------------------------------------

def cfg_single_head_fp32() -> Problem:
    """fp32, B=1, H=1, Sq=Sk=128, D=64, non-causal, scale 1/8; seed 0."""
    return batched(0, 1, 128, 128, 1, 1, 64, "f32", False, 1.0 / math.sqrt(64),
                   name="single_head_fp32_b1_h1_s128_d64")


def cfg_batched_causal(B: int = 4, S: int = 2048, H: int = 16, D: int = 128, dtype: str = "bf16") -> Problem:
    """bf16, B=4, Hq=Hkv=16, Sq=Sk=2048, D=128, causal, default scale; seed 1."""
    return batched(1, B, S, S, H, H, D, dtype, True, None,
                   name=f"batched_causal_b{B}_h{H}_s{S}_d{D}_{dtype}")


def varlen_lengths(seed: int = 2, n: int = 16, lo: int = 128, hi: int = 4096) -> tuple[torch.Generator, list[int]]:
    g = torch.Generator("cpu").manual_seed(seed)
    lens = torch.randint(lo, hi + 1, (n,), generator=g).tolist()
    return g, lens


def cfg_varlen_gqa() -> Problem:
    """bf16 varlen GQA causal: 16 sequences, lengths U[128, 4096] (seed 2),
    cu_seqlens_q = cu_seqlens_k, Hq=32, Hkv=8, D=128; q,k,v drawn from the
    same generator right after the lengths."""
    g, lens = varlen_lengths()
    t = sum(lens)
    q = _randn(g, (t, 32, 128), "bf16")
    k = _randn(g, (t, 8, 128), "bf16")
    v = _randn(g, (t, 8, 128), "bf16")
    cu = _cu(lens)
    return Problem("varlen_gqa_causal_16seq_hq32_hkv8_d128_bf16", "bf16", q, k, v, cu, cu.clone(),
                   32, 8, 128, 128, True, 128 ** -0.5, meta={"lens": lens})


def cfg_mla_decode() -> Problem:
    """MLA split-KV decode, bf16: batch 128, q_len 4, 16 heads, 576/512, kv_len 8192; seed 3."""
    return mla_decode(3, 128, 4, 8192, name="mla_decode_b128_q4_h16_kv8192_bf16")


def cfg_mla_decode_fp8() -> Problem:
    """The same MLA decode shape over an E4M3 cache (bf16 q and output); seed 3."""
    return mla_decode_fp8(3, 128, 4, 8192, name="mla_decode_b128_q4_h16_kv8192_fp8kv")


def kvcache(seed: int, batch: int, Sq: int, Snew: int, seqlens: list[int], hq: int = 32, hkv: int = 4,
            d: int = 128, dtype: str = "bf16", page_size: int | None = None, cache_len: int = 0,
            causal: bool = False) -> dict:
    """A KV-cache decode (mxflashattn flash_attn_with_kvcache): q [B, Sq, Hq, D],
    a dense cache [B, cache_len, Hkv, D] (page_size None) or a paged one
    [pages, page_size, Hkv, D] whose block table is a seeded permutation of
    the pages, cache_seqlens, and rows k_new / v_new [B, Snew, Hkv, D].  Every
    cache slot is filled with random values, so a key read past a sequence's
    length shows up in the result.  Returns the device-independent tensors and
    the equivalent packed Problem (keys in order, appended rows after the
    cached ones) for the reference computation."""
    g = torch.Generator("cpu").manual_seed(seed)
    lens = [L + Snew for L in seqlens]
    q = _randn(g, (batch, Sq, hq, d), dtype)
    k_new = _randn(g, (batch, Snew, hkv, d), dtype) if Snew else None
    v_new = _randn(g, (batch, Snew, hkv, d), dtype) if Snew else None
    if page_size is None:
        cap = max(cache_len, max(lens))
        kc = _randn(g, (batch, cap, hkv, d), dtype)
        vc = _randn(g, (batch, cap, hkv, d), dtype)
        table = None
        rows = lambda b, pos: (b, pos)
    else:
        per = [(L + page_size - 1) // page_size for L in lens]
        max_blocks = max(1, max(per))
        pages = sum(per) + 3  # a few pages no sequence uses
        kc = _randn(g, (pages, page_size, hkv, d), dtype)
        vc = _randn(g, (pages, page_size, hkv, d), dtype)
        perm = torch.randperm(pages, generator=g).tolist()
        table = torch.full((batch, max_blocks), -1, dtype=torch.int32)
        it = iter(perm)
        for b in range(batch):
            for i in range(per[b]):
                table[b, i] = next(it)
        rows = lambda b, pos: (int(table[b, pos // page_size]), pos % page_size)
    # the logical keys of each entry after the append
    ks, vs = [], []
    for b in range(batch):
        kb = torch.empty((lens[b], hkv, d), dtype=kc.dtype)
        vb = torch.empty((lens[b], hkv, d), dtype=vc.dtype)
        for pos in range(lens[b]):
            if pos < seqlens[b]:
                pg, off = rows(b, pos)
                kb[pos], vb[pos] = kc[pg, off], vc[pg, off]
            else:
                kb[pos], vb[pos] = k_new[b, pos - seqlens[b]], v_new[b, pos - seqlens[b]]
        ks.append(kb)
        vs.append(vb)
    prob = Problem(f"kvcache_b{batch}_sq{Sq}_new{Snew}", dtype, q.reshape(batch * Sq, hq, d), torch.cat(ks),
                   torch.cat(vs), _cu([Sq] * batch), _cu(lens), hq, hkv, d, d, causal, d ** -0.5)
    return {"q": q, "k_cache": kc, "v_cache": vc, "k_new": k_new, "v_new": v_new,
            "cache_seqlens": torch.tensor(seqlens, dtype=torch.int32), "block_table": table, "rows": rows,
            "lens": lens, "problem": prob}


def cfg_gqa_decode(batch: int = 64, kv_len: int = 8192) -> Problem:
    """Grouped-query decode (next scope row): q_len 1, Hq 32, Hkv 4, D 128,
    bf16, kv_len 8192 per sequence, seed 6; KV 1.07 GB, larger than L2."""
    return gqa_decode(6, batch, 1, kv_len)


def cfg_long_causal(S: int = 32768, H: int = 32, rows_per_head: int = 256) -> Problem:
    """bf16, B=1, Hq=Hkv=32, Sq=Sk=32768, D=128, causal; seed 4. After q,k,v the
    same generator draws randperm(S)[:256] per head; rows 0 and S-1 are added."""
    g = torch.Generator("cpu").manual_seed(4)
    q = _randn(g, (S, H, 128), "bf16")
    k = _randn(g, (S, H, 128), "bf16")
    v = _randn(g, (S, H, 128), "bf16")
    pairs = []
    for h in range(H):
        rows = torch.randperm(S, generator=g)[:rows_per_head].tolist()
        for r in sorted(set(rows) | {0, S - 1}):
            pairs.append((r, h))
    cu = _cu([S])
    return Problem(f"long_causal_b1_h{H}_s{S}_d128_bf16", "bf16", q, k, v, cu, cu.clone(), H, H, 128, 128,
                   True, 128 ** -0.5, batched=True, check_rows=torch.tensor(pairs, dtype=torch.int64),
                   meta={"B": 1, "Sq": S, "Sk": S})


def to_device(p: Problem, device="cuda") -> dict:
    """The problem's tensors copied to `device` (a plain copy, no arithmetic):
    q, k, v, cu_q, cu_k, and for MLA decode the one kv cache with k and v as
    its [total, 1, 576] and [total, 1, 512] views."""
    d = {"q": p.q.to(device), "k": p.k.to(device), "v": p.v.to(device),
         "cu_q": p.cu_q.to(device), "cu_k": p.cu_k.to(device)}
    if p.mla:
        d["kv"] = p.kv.to(device)
        d["k"] = d["kv"].view(-1, 1, p.dqk)
        d["v"] = d["kv"][:, :p.dv].view(-1, 1, p.dv)
    return d


def sample_rows(p: Problem, n_per_head: int, seed: int) -> torch.Tensor:
    """(token, head) pairs for a sampled oracle check: n random tokens per head,
    plus the first and last token of every sequence."""
    g = torch.Generator("cpu").manual_seed(seed)
    ends = set()
    c = p.cu_q.tolist()
    for b in range(p.batch):
        if c[b + 1] > c[b]:
            ends |= {c[b], c[b + 1] - 1}
    pairs = []
    for h in range(p.hq):
        rows = torch.randint(0, p.total_q, (n_per_head,), generator=g).tolist()
        for r in sorted(set(rows) | ends):
            pairs.append((r, h))
    return torch.tensor(pairs, dtype=torch.int64)
