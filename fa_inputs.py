"""Seeded synthetic inputs for the attention forward workloads.

Shared by the tests, the smoke check and the benchmark.  It holds no attention
arithmetic: it only draws Q/K/V/bias tensors and sequence-length metadata from
a seeded generator, plus the algorithmic work counts used to report
throughput.  Both the CUDA path and the oracle read the same bits from here.

Workloads (shapes from the pages' validation tables and API contracts):

* ``dense_257``: dense non-causal MHA, B=1, S=257, H=8, D=128 (the small bf16
  validation shape of "FlashAttention-4", GB10 Validation).
* ``varlen_gqa_bias``: varlen causal GQA 32/8, D=128, 4 sequences with lengths
  uniform in [512, 4096], rel_bias [total_q, 32, 256] ~ N(0, 0.5^2)
  ("mgoin/tml-fa4", argument contract).
* ``video_dit_20480``: dense non-causal MHA, B=1, S=20480, H=56, D=128 (the
  long bf16 validation shape of "FlashAttention-4", GB10 Validation).
* ``encoder_d256_seqused``: GQA 8/1, D=256, B=2, Sq=1024, K/V padded to 1024
  with seqused_k=968; padded K/V rows hold 1e4 so that a masking error shows
  ("flashrt/fa4-cute-runtime", forward_static with seqused_k).
* ``decode_splitkv``: B=8, Sq=1, Sk=131072, Hq=32, Hkv=8, D=128 split-KV
  decode with an LSE combine.
* ``dense_d64``: dense non-causal MHA, B=4, S=4096, H=16, D=64 (a 64-wide
  head dim, one of the small head dims the pages list as the next step).
* ``local_window_softcap``: causal GQA 16/4, D=128, B=1, S=32768 with a
  sliding window of 4095 keys to the left and scores soft-capped at 50 (the
  pages' "mask/score modifiers", at local-attention sizes).
* ``tabpfn_d16``: dense non-causal MHA, fp16, B=1, S=30000, H=8, D=16: the
  head-dim-16 attention stages of "FlashAttention-4 backend for Blackwell
  #1235" (keys = n_train, here the 30k rows from which the issue reports
  gains; fp16 as its autocast; the head count is not given: 8).
* ``vision_d72``: dense non-causal MHA, B=32, S=729, H=16, D=72: the D72 MHA
  profile of "flashrt/fa4-cute-runtime" (a vision encoder; the page gives no
  shape: 27x27 patches, 16 heads, a batch of 32 images).
* ``dense_d256``: dense non-causal MHA, B=4, S=4096, H=8, D=256: a head-dim-256
  problem of several waves of 256-row units (the D256 path of
  "flashrt/fa4-cute-runtime" at a size where the key loop dominates; the page
  gives no shape).

Seeds are 440410 + workload index (the seed style of the pages' benchmark).
Values are drawn in float32 as N(0, 1) and rounded to the input dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

SEED_BASE = 440410

WORKLOADS = ["dense_257", "varlen_gqa_bias", "video_dit_20480",
             "encoder_d256_seqused", "decode_splitkv", "dense_d64",
             "local_window_softcap", "tabpfn_d16", "vision_d72", "dense_d256"]

_CHUNK = 1 << 24


def _randn(shape, gen: torch.Generator, dtype, std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) in float32, rounded to ``dtype``, drawn in chunks on the
    generator's device."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=dtype, device=gen.device)
    for start in range(0, n, _CHUNK):
        m = min(_CHUNK, n - start)
        x = torch.randn(m, generator=gen, dtype=torch.float32, device=gen.device)
        if std != 1.0:
            x.mul_(std)
        out[start:start + m].copy_(x)
    return out.view(*shape)


@dataclass
class Problem:
    """One attention forward problem, CPU tensors unless moved."""
    name: str
    layout: str                      # "dense" or "varlen"
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    causal: bool = False
    softmax_scale: Optional[float] = None
    cu_seqlens_q: Optional[torch.Tensor] = None
    cu_seqlens_k: Optional[torch.Tensor] = None
    seqused_k: Optional[torch.Tensor] = None
    rel_bias: Optional[torch.Tensor] = None
    max_seqlen_q: int = 0
    max_seqlen_k: int = 0
    splitkv: bool = False
    meta: dict = field(default_factory=dict)
    window: tuple = (-1, -1)         # (left, right) bounds by diagonal distance; < 0: none
    softcap: float = 0.0             # > 0: scores capped as softcap * tanh(s / softcap)

    # -- shapes -----------------------------------------------------------
    @property
    def D(self) -> int:
        return int(self.q.shape[-1])

    @property
    def Hq(self) -> int:
        return int(self.q.shape[-2])

    @property
    def Hkv(self) -> int:
        return int(self.k.shape[-2])

    @property
    def B(self) -> int:
        if self.layout == "dense":
            return int(self.q.shape[0])
        return int(self.cu_seqlens_q.shape[0]) - 1

    def seq_lens(self):
        """[(q_len, k_len_used)] per batch entry, as plain ints."""
        if self.layout == "dense":
            Sq, Sk = int(self.q.shape[1]), int(self.k.shape[1])
            lens = [(Sq, Sk)] * self.B
        else:
            cq = self.cu_seqlens_q.tolist()
            ck = self.cu_seqlens_k.tolist()
            lens = [(cq[b + 1] - cq[b], ck[b + 1] - ck[b])
                    for b in range(self.B)]
        if self.seqused_k is not None:
            su = self.seqused_k.tolist()
            lens = [(ql, su[b]) for b, (ql, _) in enumerate(lens)]
        return lens

    # -- algorithmic work (the metric's definition) ------------------------
    def admitted_keys(self, ql: int, kl: int, i: int) -> int:
        """Keys row i of a (q_len, k_len) sequence attends to under the
        causal flag and the window (distance d = i + kl - ql - j)."""
        delta = kl - ql
        lo, hi = 0, kl - 1
        wl, wr = self.window
        if self.causal:
            wr = 0 if wr < 0 else min(wr, 0)
        if wr >= 0:
            hi = min(hi, i + delta + wr)
        if wl >= 0:
            lo = max(lo, i + delta - wl)
        return max(0, hi - lo + 1)

    def flops(self) -> float:
        """4 * q_len * k_len * D * Hq per sequence, halved when causal; with a
        window, 4 * D * Hq per admitted (row, key) pair."""
        f = 0.0
        if self.window[0] >= 0 or self.window[1] >= 0:
            for ql, kl in self.seq_lens():
                f += 4.0 * self.D * self.Hq * sum(self.admitted_keys(ql, kl, i) for i in range(ql))
            return f
        for ql, kl in self.seq_lens():
            f += 4.0 * ql * kl * self.D * self.Hq
        return f * (0.5 if self.causal else 1.0)

    def hbm_bytes(self) -> float:
        """Bytes the unsplit operation must move: K, V (used rows), Q, O, LSE
        and the bias tensor when present."""
        es = self.q.element_size()
        tq = sum(ql for ql, _ in self.seq_lens())
        tk = sum(kl for _, kl in self.seq_lens())
        b = 2.0 * tk * self.Hkv * self.D * es          # K and V
        b += 2.0 * tq * self.Hq * self.D * es          # Q and O
        b += 4.0 * tq * self.Hq                        # LSE
        if self.rel_bias is not None:
            b += self.rel_bias.numel() * es
        return b

    def to(self, device) -> "Problem":
        kw = {}
        for name in ("q", "k", "v", "cu_seqlens_q", "cu_seqlens_k",
                     "seqused_k", "rel_bias"):
            t = getattr(self, name)
            kw[name] = None if t is None else t.to(device)
        return Problem(self.name, self.layout, kw["q"], kw["k"], kw["v"],
                       self.causal, self.softmax_scale, kw["cu_seqlens_q"],
                       kw["cu_seqlens_k"], kw["seqused_k"], kw["rel_bias"],
                       self.max_seqlen_q, self.max_seqlen_k, self.splitkv,
                       dict(self.meta), tuple(self.window), self.softcap)


def make(name: str, dtype=torch.bfloat16, device="cpu", decode_sk: int = 131072,
         dit_s: int = 20480) -> Problem:
    """Build one named workload with its fixed seed.

    With ``device`` other than the CPU the values are drawn there by that
    device's seeded generator (another stream of numbers than the CPU
    generator's, same distributions and shapes): the benchmark uses this for
    the multi-GB workloads; parity tests draw on the CPU.  ``decode_sk``
    shortens the decode workload's keys and ``dit_s`` the video workload's
    sequence (for profiling a smaller case)."""
    idx = WORKLOADS.index(name)
    g = torch.Generator(device=device).manual_seed(SEED_BASE + idx)
    if name == "dense_257":
        B, S, H, D = 1, 257, 8, 128
        q = _randn((B, S, H, D), g, dtype)
        k = _randn((B, S, H, D), g, dtype)
        v = _randn((B, S, H, D), g, dtype)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=S, max_seqlen_k=S)
    if name == "varlen_gqa_bias":
        Hq, Hkv, D, R = 32, 8, 128, 256
        lens = torch.randint(512, 4097, (4,), generator=g, device=g.device).tolist()
        cu = torch.tensor([0] + list(_cumsum(lens)), dtype=torch.int32, device=g.device)
        total = int(cu[-1])
        q = _randn((total, Hq, D), g, dtype)
        k = _randn((total, Hkv, D), g, dtype)
        v = _randn((total, Hkv, D), g, dtype)
        rb = _randn((total, Hq, R), g, dtype, std=0.5)
        return Problem(name, "varlen", q, k, v, causal=True,
                       softmax_scale=1 / math.sqrt(D), cu_seqlens_q=cu,
                       cu_seqlens_k=cu.clone(), rel_bias=rb,
                       max_seqlen_q=max(lens), max_seqlen_k=max(lens),
                       meta={"lens": lens})
    if name == "video_dit_20480":
        B, S, H, D = 1, int(dit_s), 56, 128
        q = _randn((B, S, H, D), g, dtype)
        k = _randn((B, S, H, D), g, dtype)
        v = _randn((B, S, H, D), g, dtype)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=S, max_seqlen_k=S)
    if name == "encoder_d256_seqused":
        B, Sq, Sk, Hq, Hkv, D, used = 2, 1024, 1024, 8, 1, 256, 968
        q = _randn((B, Sq, Hq, D), g, dtype)
        k = _randn((B, Sk, Hkv, D), g, dtype)
        v = _randn((B, Sk, Hkv, D), g, dtype)
        k[:, used:] = 1e4
        v[:, used:] = 1e4
        su = torch.full((B,), used, dtype=torch.int32, device=g.device)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       seqused_k=su, max_seqlen_q=Sq, max_seqlen_k=Sk)
    if name == "decode_splitkv":
        B, Sq, Sk, Hq, Hkv, D = 8, 1, int(decode_sk), 32, 8, 128
        q = _randn((B, Sq, Hq, D), g, dtype)
        k = _randn((B, Sk, Hkv, D), g, dtype)
        v = _randn((B, Sk, Hkv, D), g, dtype)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=Sq, max_seqlen_k=Sk, splitkv=True)
    if name == "dense_d64":
        B, S, H, D = 4, 4096, 16, 64
        q = _randn((B, S, H, D), g, dtype)
        k = _randn((B, S, H, D), g, dtype)
        v = _randn((B, S, H, D), g, dtype)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=S, max_seqlen_k=S)
    if name == "local_window_softcap":
        B, S, Hq, Hkv, D = 1, 32768, 16, 4, 128
        q = _randn((B, S, Hq, D), g, dtype)
        k = _randn((B, S, Hkv, D), g, dtype)
        v = _randn((B, S, Hkv, D), g, dtype)
        return Problem(name, "dense", q, k, v, causal=True, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=S, max_seqlen_k=S, window=(4095, -1), softcap=50.0)
    if name == "tabpfn_d16":
        B, S, H, D = 1, 30000, 8, 16
        q = _randn((B, S, H, D), g, torch.float16)
        k = _randn((B, S, H, D), g, torch.float16)
        v = _randn((B, S, H, D), g, torch.float16)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=S, max_seqlen_k=S)
    if name == "vision_d72":
        B, S, H, D = 32, 729, 16, 72
        q = _randn((B, S, H, D), g, dtype)
        k = _randn((B, S, H, D), g, dtype)
        v = _randn((B, S, H, D), g, dtype)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=S, max_seqlen_k=S)
    if name == "dense_d256":
        B, S, H, D = 4, 4096, 8, 256
        q = _randn((B, S, H, D), g, dtype)
        k = _randn((B, S, H, D), g, dtype)
        v = _randn((B, S, H, D), g, dtype)
        return Problem(name, "dense", q, k, v, softmax_scale=1 / math.sqrt(D),
                       max_seqlen_q=S, max_seqlen_k=S)
    raise KeyError(name)


def _cumsum(xs):
    s = 0
    for x in xs:
        s += x
        yield s


def random_dense(seed: int, B: int, Sq: int, Sk: int, Hq: int, Hkv: int,
                 D: int, dtype=torch.bfloat16, causal=False, seqused=None,
                 pad_value=None, bias_extent: int = 0, bias_std: float = 0.5,
                 q_std: float = 1.0, v_offset: float = 0.0) -> Problem:
    """A dense problem of any shape, for parity and edge-case tests.

    ``seqused`` (list of ints) marks the valid K/V rows per batch entry;
    ``pad_value`` fills the rest.  ``q_std`` sharpens the softmax and
    ``v_offset`` shifts V away from zero (stress inputs).
    """
    g = torch.Generator().manual_seed(seed)
    q = _randn((B, Sq, Hq, D), g, dtype, std=q_std)
    k = _randn((B, Sk, Hkv, D), g, dtype)
    v = _randn((B, Sk, Hkv, D), g, dtype)
    if v_offset:
        v = (v.float() + v_offset).to(dtype)
    su = None
    if seqused is not None:
        su = torch.tensor(seqused, dtype=torch.int32)
        if pad_value is not None:
            for b, u in enumerate(seqused):
                k[b, u:] = pad_value
                v[b, u:] = pad_value
    rb = None
    if bias_extent:
        rb = _randn((B, Sq, Hq, bias_extent), g, dtype, std=bias_std)
    return Problem(f"dense_{seed}", "dense", q, k, v, causal=causal,
                   seqused_k=su, rel_bias=rb, max_seqlen_q=Sq,
                   max_seqlen_k=Sk)


def random_varlen(seed: int, q_lens, k_lens, Hq: int, Hkv: int, D: int,
                  dtype=torch.bfloat16, causal=False, bias_extent: int = 0,
                  bias_std: float = 0.5, seqused=None) -> Problem:
    """A varlen problem with the given per-sequence lengths."""
    g = torch.Generator().manual_seed(seed)
    cu_q = torch.tensor([0] + list(_cumsum(q_lens)), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(_cumsum(k_lens)), dtype=torch.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = _randn((tq, Hq, D), g, dtype)
    k = _randn((tk, Hkv, D), g, dtype)
    v = _randn((tk, Hkv, D), g, dtype)
    rb = None
    if bias_extent:
        rb = _randn((tq, Hq, bias_extent), g, dtype, std=bias_std)
    su = None if seqused is None else torch.tensor(seqused, dtype=torch.int32)
    return Problem(f"varlen_{seed}", "varlen", q, k, v, causal=causal,
                   cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, seqused_k=su,
                   rel_bias=rb, max_seqlen_q=max(q_lens, default=0),
                   max_seqlen_k=max(k_lens, default=0))
