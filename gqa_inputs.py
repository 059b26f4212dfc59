"""Seeded synthetic inputs for the GQA prefill and decode workloads.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It only draws random numbers and describes shapes; it contains none of the
attention arithmetic (no RoPE, no scores, no softmax), so that the oracle and
the CUDA path share nothing but their inputs.

Recipe (one seed per workload, ``seed = 1000 + workload index``):
  * Q, K, V (and the decode caches) are drawn as float32 N(0, 1) from a
    ``torch.Generator`` seeded with the workload's seed, in the order
    q, k, v (prefill) or seqlens, q, kcache, vcache (decode), then rounded to
    bfloat16 (round to nearest even).
  * Decode cache lengths are uniform integers in [1, max_len].
  * Shapes are the Qwen2 model shapes of the page "Qwen2 architecture
    introduction" (aicoding.csdn.net), §4.4 Table 1: 0.5B 14/2 heads with head
    size 64, 7B 28/4 heads with head size 128, 72B 64/8 heads with head size 128;
    RoPE base 1e6 (same page, §5.2).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

THETA = 1.0e6


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    B: int
    h_q: int
    h_kv: int
    d: int
    L: int = 0           # prefill sequence length
    max_len: int = 0     # decode: cache lengths are uniform in [1, max_len]
    theta: float = THETA
    seed: int = 0
    desc: str = field(default="", compare=False)

    @property
    def g(self) -> int:
        return self.h_q // self.h_kv

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads, in their canonical order (the index fixes the seed).
WORKLOADS = [
    Workload("qwen2-0.5b-prefill-L128", "prefill", B=1, L=128, h_q=14, h_kv=2, d=64,
             desc="Qwen2-0.5B-shaped single-layer GQA prefill, B=1 L=128 h_q=14 h_kv=2 d=64"),
    Workload("qwen2-7b-prefill-L4096", "prefill", B=1, L=4096, h_q=28, h_kv=4, d=128,
             desc="Qwen2-7B-shaped GQA prefill, B=1 L=4096 h_q=28 h_kv=4 d=128"),
    Workload("qwen2-72b-prefill-B4-L8192", "prefill", B=4, L=8192, h_q=64, h_kv=8, d=128,
             desc="Qwen2-72B-shaped GQA prefill, B=4 L=8192 h_q=64 h_kv=8 d=128"),
    Workload("qwen2-7b-decode-B64", "decode", B=64, max_len=32768, h_q=28, h_kv=4, d=128,
             desc="Qwen2-7B-shaped GQA decode, B=64, cache lengths uniform in [1, 32768], h_q=28 h_kv=4 d=128"),
    Workload("qwen2-7b-prefill-L32768", "prefill", B=1, L=32768, h_q=28, h_kv=4, d=128,
             desc="Qwen2-7B-shaped long-context GQA prefill, B=1 L=32768 h_q=28 h_kv=4 d=128"),
]
WORKLOADS = [w.with_(seed=1000 + i) for i, w in enumerate(WORKLOADS)]
BY_NAME = {w.name: w for w in WORKLOADS}


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, gen, device="cpu", chunk_rows=1 << 16):
    """N(0,1) float32 rounded to bf16; drawn in leading-dim chunks to bound host memory."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    n0 = shape[0]
    for s in range(0, n0, chunk_rows):
        e = min(n0, s + chunk_rows)
        out[s:e] = torch.randn((e - s,) + tuple(shape[1:]), generator=gen,
                               dtype=torch.float32, device=device).to(torch.bfloat16)
    return out


def prefill_inputs(w: Workload, device: str = "cpu"):
    """q [B,L,h_q,d], k [B,L,h_kv,d], v [B,L,h_kv,d], all bf16, token-major."""
    assert w.kind == "prefill"
    gen = _gen(w.seed, device)
    q = _randn_bf16((w.B * w.L, w.h_q, w.d), gen, device).view(w.B, w.L, w.h_q, w.d)
    k = _randn_bf16((w.B * w.L, w.h_kv, w.d), gen, device).view(w.B, w.L, w.h_kv, w.d)
    v = _randn_bf16((w.B * w.L, w.h_kv, w.d), gen, device).view(w.B, w.L, w.h_kv, w.d)
    return q, k, v


# Hidden size of the Qwen2 models whose head shapes the workloads use (Qwen2-0.5B: 896, Qwen2-7B: 3584,
# Qwen2-72B: 8192): the K dimension of the fused QKV projection.
D_MODEL = {(14, 2, 64): 896, (28, 4, 128): 3584, (64, 8, 128): 8192}


def qkv_inputs(w: Workload, d_model: int | None = None, device: str = "cpu", bias: bool = True):
    """Synthetic inputs of the fused QKV projection for the prefill workload w.

    x [B, L, d_model] ~ N(0, 1) (hidden states after RMSNorm); w_qkv [(h_q + 2 h_kv) d, d_model]
    ~ N(0, 1/d_model), the rows of W_Q^T, W_K^T, W_V^T stacked (the nn.Linear weight layout);
    b_qkv [(h_q + 2 h_kv) d] ~ N(0, 0.1^2) or None.  All bf16.  The weight scale keeps projected values
    near unit size, as in trained models.
    """
    assert w.kind == "prefill"
    dm = d_model or D_MODEL[(w.h_q, w.h_kv, w.d)]
    n = (w.h_q + 2 * w.h_kv) * w.d
    gen = _gen(w.seed + 31337, device)
    x = _randn_bf16((w.B * w.L, dm), gen, device).view(w.B, w.L, dm)
    wq = torch.empty((n, dm), dtype=torch.bfloat16, device=device)
    for s0 in range(0, n, 1024):
        e = min(n, s0 + 1024)
        wq[s0:e] = (torch.randn((e - s0, dm), generator=gen, dtype=torch.float32, device=device)
                    / (dm ** 0.5)).to(torch.bfloat16)
    b = None
    if bias:
        b = (0.1 * torch.randn((n,), generator=gen, dtype=torch.float32, device=device)).to(torch.bfloat16)
    return x, wq, b


def out_proj_inputs(w: Workload, d_model: int | None = None, device: str = "cpu"):
    """Synthetic inputs of the output projection for the prefill workload w: attn [B*L, h_q*d] ~ N(0, 1)
    (the concatenated heads), w_o [d_model, h_q*d] ~ N(0, 1/(h_q*d)) (nn.Linear layout), residual
    [B*L, d_model] ~ N(0, 1).  All bf16."""
    assert w.kind == "prefill"
    dm = d_model or D_MODEL[(w.h_q, w.h_kv, w.d)]
    k = w.h_q * w.d
    gen = _gen(w.seed + 4242, device)
    attn = _randn_bf16((w.B * w.L, k), gen, device)
    wo = torch.empty((dm, k), dtype=torch.bfloat16, device=device)
    for s0 in range(0, dm, 1024):
        e = min(dm, s0 + 1024)
        wo[s0:e] = (torch.randn((e - s0, k), generator=gen, dtype=torch.float32, device=device)
                    / (k ** 0.5)).to(torch.bfloat16)
    res = _randn_bf16((w.B * w.L, dm), gen, device)
    return attn, wo, res


def decode_inputs(w: Workload, device: str = "cpu", seqlens=None):
    """seqlens int32 [B]; q [B,h_q,d]; kcache, vcache packed [sum(seqlens), h_kv, d].

    Sequence b's cache rows sit at packed rows off_b .. off_b + seqlens[b] - 1,
    with off_b the sum of the lengths before it. ``seqlens`` may be given to
    override the drawn lengths (edge-case tests); the draw still happens so the
    random stream stays the same.
    """
    assert w.kind == "decode"
    gen = _gen(w.seed, device)
    drawn = torch.randint(1, w.max_len + 1, (w.B,), generator=gen, dtype=torch.int64,
                          device=device).to(torch.int32)
    if seqlens is not None:
        drawn = torch.as_tensor(seqlens, dtype=torch.int32, device=device)
        assert drawn.numel() == w.B
    total = int(drawn.sum().item())
    q = _randn_bf16((w.B, w.h_q, w.d), gen, device)
    kc = _randn_bf16((max(total, 0), w.h_kv, w.d), gen, device)
    vc = _randn_bf16((max(total, 0), w.h_kv, w.d), gen, device)
    return drawn, q, kc, vc


def paged_layout(seqlens, page_size: int, seed: int, extra_pages: int = 3, max_pages: int | None = None,
                 device: str = "cpu"):
    """A seeded paged placement of sequences of the given lengths (storage layout only).

    Each sequence b needs ceil(seqlens[b] / page_size) pages; all needed pages plus `extra_pages`
    unused ones are numbered in a random order, so neighbouring pages of a sequence are scattered.
    Returns (block_table int32 [B, max_pages], num_pages, store_row int64 [sum(seqlens)]), where
    block_table[b, i] is the page of the i-th block of sequence b (-1 past its last page) and
    store_row[off_b + j] = page * page_size + j % page_size is where packed row off_b + j lives.
    """
    lens = [int(x) for x in torch.as_tensor(seqlens).tolist()]
    need = [(n + page_size - 1) // page_size for n in lens]
    num_pages = sum(need) + extra_pages
    mp = max(need + [1]) if max_pages is None else max_pages
    perm = torch.randperm(num_pages, generator=_gen(seed, "cpu")).to(torch.int32)
    table = torch.full((len(lens), mp), -1, dtype=torch.int32)
    rows = []
    nxt = 0
    for b, (n, k) in enumerate(zip(lens, need)):
        table[b, :k] = perm[nxt:nxt + k]
        nxt += k
        j = torch.arange(n, dtype=torch.int64)
        rows.append(table[b, (j // page_size)].to(torch.int64) * page_size + j % page_size)
    store_row = torch.cat(rows) if rows else torch.zeros(0, dtype=torch.int64)
    return table.to(device), num_pages, store_row.to(device)


def decode_paged_inputs(w: Workload, page_size: int, device: str = "cpu", seqlens=None, extra_pages: int = 3):
    """decode_inputs(w) with the packed caches scattered into pages.

    Returns seqlens, q, kpages, vpages [num_pages, page_size, h_kv, d], block_table [B, max_pages],
    num_pages, and the packed caches themselves.  Page slots that hold no cache row are filled with
    N(0,1) values, so a wrong slot read shows up in the result.
    """
    s, q, kc, vc = decode_inputs(w, device, seqlens=seqlens)
    table, num_pages, store_row = paged_layout(s.cpu(), page_size, w.seed + 7919, extra_pages, device=device)
    gen = _gen(w.seed + 104729, device)
    kp = _randn_bf16((num_pages * page_size, w.h_kv, w.d), gen, device)
    vp = _randn_bf16((num_pages * page_size, w.h_kv, w.d), gen, device)
    kp[store_row] = kc
    vp[store_row] = vc
    shape = (num_pages, page_size, w.h_kv, w.d)
    return s, q, kp.view(shape), vp.view(shape), table, num_pages, kc, vc


def small(kind: str, B: int, h_q: int, h_kv: int, d: int, L: int = 0, max_len: int = 0,
          seed: int = 7, theta: float = THETA, name: str = "") -> Workload:
    """A small ad-hoc workload for tests (ragged sizes, special head counts)."""
    return Workload(name or f"{kind}-B{B}-L{L or max_len}-hq{h_q}-hkv{h_kv}-d{d}", kind,
                    B=B, L=L, max_len=max_len, h_q=h_q, h_kv=h_kv, d=d, theta=theta, seed=seed)
