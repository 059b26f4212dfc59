"""Plain fp64 CPU oracle for Qwen2-style grouped-query causal self-attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` use it.  It shares no code
with the CUDA library; the two meet only through the seeded inputs of
``gqa_inputs``.

What it computes is the textbook definition, written out step by step in
float64 with NumPy, with no blocking or fusion beyond splitting the query rows
into independent blocks (each block is still the full materialised product):

  1. RoPE on Q and K (page "Qwen2架构解析：GQA与MoE技术在大模型中的创新应用",
     intelliparadigm.com, §2.3; page "Qwen2 architecture introduction",
     aicoding.csdn.net, §3.5.2 and §4.1.3 step 3): every Q and K row at
     position m is rotated, pair by pair, by the angle m * theta^(-2i/d),
     with d the head size and theta the RoPE base (1e6, same page §5.2).
     Pairing: dimension i with i + d/2 ("rotate half"); the rotation is the
     ordinary positive-angle plane rotation, i.e. the complex product
     (x_i + j x_{i+d/2}) * exp(j * m * theta^(-2i/d)).
  2. Head grouping (aicoding.csdn.net page, §4.1.2): with g = h_q / h_kv,
     query head t (1-based) reads KV group floor((t-1)/g) + 1; 0-based this is
     u = t // g.
  3. Scores, mask, softmax, weighted sum (aicoding.csdn.net page, §4.1.3
     step 4): S = Q' K'^T / sqrt(d), S_ij = -inf where j > i, A = row softmax,
     head_t = A V_u.  The output keeps the concatenated-heads layout of §4.1.3
     step 5: out[b, i, t, :] is row i of head_t.
  4. Decode (aicoding.csdn.net page, §4.1.3 closing paragraph; page "从 Qwen 1
     到 Qwen 2", nxmr.cn, §2.4): the cache holds only the h_kv groups of
     un-rotated K and V; one new query per sequence, at position
     p = seqlens[b], attends to all seqlens[b] cached rows (positions
     0 .. p-1).  ``include_self=True`` selects the other reading, where the
     cache already holds the new token and the query sits at p - 1.
  5. Paged cache (nxmr.cn page, §2.4: PagedAttention keeps the cache of each
     KV head in fixed-size blocks): the same decode, with position j of
     sequence b read from slot j % page_size of page block_table[b, j //
     page_size].  ``decode_paged_ref`` gathers the rows and applies step 4.
     ``qkv_append_ref`` is one decode step's projection: the new token's q,
     and its k, v written into the page slot of position seqlens[b] (the
     cache grows by the current token each step, aicoding.csdn.net page,
     §4.1.3 closing paragraph).
  6. QKV projection (aicoding.csdn.net page, §4.1.3 steps 1-3): Q, K, V are
     the hidden states times W_Q, W_K, W_V plus the bias, split into h_q and
     h_kv heads; Q and K are then rotated as in step 1.
     ``qkv_rope_ref`` writes it out with one matrix product.
  7. Output projection and residual (aicoding.csdn.net page, §4.1.3 steps
     5-6): the concatenated heads times W_O, plus the sub-layer input.
     ``out_proj_ref``.
  8. YaRN scaling of RoPE for contexts beyond the trained window (yudonglee.me
     page, §6.2: per-dimension interpolation f_i / s * alpha_i with a ramp
     alpha_i; aicoding.csdn.net page, §5.3: a length-dependent rescaling of
     the attention logits).  The pages give neither the ramp's bounds nor
     the rescaling formula; ``Yarn`` takes the published YaRN method's
     (turn-count bounds 1 and 32, temperature (0.1 ln s + 1)^2).  Parity
     unpinned by the pages for those constants: the pins fix only the
     form (factor 1 = plain RoPE, fast pairs kept, slow pairs divided by s,
     logits rescaled).  Pass a ``Yarn`` wherever ``theta`` is taken.

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
invariants the pages state and a brute-force restatement.
"""
from __future__ import annotations

from typing import NamedTuple

import numpy as np


def as_f64(x) -> np.ndarray:
    """Upcast a torch tensor (any float dtype, CPU) or array to a float64 ndarray."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def head_group(t: int, g: int) -> int:
    """0-based KV group of 0-based query head t (aicoding.csdn.net page, §4.1.2)."""
    return t // g


class Yarn(NamedTuple):
    """A RoPE base with YaRN scaling, usable wherever a plain base `theta` is (step 8 of the module
    docstring).  factor s = 1 is plain RoPE."""
    base: float
    factor: float
    original_max: int
    beta_fast: float = 32.0
    beta_slow: float = 1.0


def inv_freq(d: int, theta) -> np.ndarray:
    """theta^(-2i/d) for i = 0 .. d/2 - 1 (intelliparadigm.com page, §2.3, with d the head size).

    With a Yarn spec (yudonglee.me page, §6.2): f'_i = f_i / s * alpha_i, where alpha_i ramps from 1 to s
    over the dimension pairs: alpha_i = 1 + gamma_i (s - 1), gamma_i = clip((r_i - beta_slow) /
    (beta_fast - beta_slow), 0, 1), r_i = original_max * f_i / (2 pi) the turns of pair i over the
    original window.  Pairs that turn many times keep their frequency; slow ones are interpolated by s.
    """
    base = theta.base if isinstance(theta, Yarn) else float(theta)
    i = np.arange(d // 2, dtype=np.float64)
    f = np.power(float(base), -2.0 * i / d)
    if isinstance(theta, Yarn) and theta.factor != 1.0:
        r = theta.original_max * f / (2.0 * np.pi)
        gamma = np.clip((r - theta.beta_slow) / (theta.beta_fast - theta.beta_slow), 0.0, 1.0)
        f = f / theta.factor * (1.0 + gamma * (theta.factor - 1.0))
    return f


def rope_mscale(theta) -> float:
    """YaRN's attention temperature as a factor on the rotated Q and K rows: 0.1 ln(s) + 1, so the scores
    scale by its square (aicoding.csdn.net page, §5.3: a length-dependent rescaling of the attention
    logits); 1 without scaling."""
    return 0.1 * np.log(theta.factor) + 1.0 if isinstance(theta, Yarn) and theta.factor > 1.0 else 1.0


def rope(x: np.ndarray, positions, theta) -> np.ndarray:
    """Rotate rows of x [..., P, H, d] at positions [P] (step 1 of the module docstring)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq(d, theta)[None, :]
    m = rope_mscale(theta)
    c = m * np.cos(ang)[:, None, :]
    s = m * np.sin(ang)[:, None, :]
    x1 = x[..., :h]
    x2 = x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_interleaved(x: np.ndarray, positions, theta: float) -> np.ndarray:
    """The other common pairing (2i with 2i+1); used only to test the permutation identity."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq(d, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xo * c + xe * s
    return out


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax with the row maximum subtracted; -inf entries get weight 0."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def causal_weights(qr_rows: np.ndarray, row_pos: np.ndarray, kr: np.ndarray) -> np.ndarray:
    """A = softmax(Q'K'^T/sqrt(d) + M) for the query rows at positions row_pos against keys 0..n-1.

    qr_rows [R, d] (rotated), kr [n, d] (rotated); M_ij = -inf where key j > query position.
    """
    d = qr_rows.shape[-1]
    s = (qr_rows @ kr.T) / np.sqrt(d)
    j = np.arange(kr.shape[0])[None, :]
    s = np.where(j > np.asarray(row_pos)[:, None], -np.inf, s)
    return softmax_rows(s)


def prefill_ref(q, k, v, theta: float, row_block: int = 1024) -> np.ndarray:
    """Full causal GQA prefill.  q [B,L,h_q,d], k/v [B,L,h_kv,d]; returns float64 [B,L,h_q,d]."""
    q = as_f64(q)
    k = as_f64(k)
    v = as_f64(v)
    B, L, h_q, d = q.shape
    h_kv = k.shape[2]
    assert h_q % h_kv == 0
    g = h_q // h_kv
    pos = np.arange(L)
    qr = rope(q, pos, theta)
    kr = rope(k, pos, theta)
    out = np.empty((B, L, h_q, d), dtype=np.float64)
    for b in range(B):
        for t in range(h_q):
            u = head_group(t, g)
            for r0 in range(0, L, row_block):
                r1 = min(L, r0 + row_block)
                rows = np.arange(r0, r1)
                a = causal_weights(qr[b, r0:r1, t, :], rows, kr[b, :r1, u, :])
                out[b, r0:r1, t, :] = a @ v[b, :r1, u, :]
    return out


def prefill_rows_ref(q, k, v, theta: float, b: int, t: int, rows) -> np.ndarray:
    """Selected output rows out[b, rows, t, :] of the causal prefill (for full-size spot checks).

    Only the key rows 0 .. max(rows) are touched, so this works at any L.
    """
    rows = np.asarray(rows, dtype=np.int64)
    h_q = q.shape[2]
    h_kv = k.shape[2]
    d = q.shape[3]
    u = head_group(t, h_q // h_kv)
    n = int(rows.max()) + 1
    qr = rope(as_f64(q[b, rows, t, :])[:, None, :], rows, theta)[:, 0, :]
    kr = rope(as_f64(k[b, :n, u, :])[:, None, :], np.arange(n), theta)[:, 0, :]
    a = causal_weights(qr, rows, kr)
    return a @ as_f64(v[b, :n, u, :])


def decode_one_ref(q_b, krows, vrows, theta: float, include_self: bool = False,
                   k_rotated: bool = False) -> np.ndarray:
    """One sequence: q_b [h_q,d], cache rows krows/vrows [s,h_kv,d] -> float64 [h_q,d].

    The cached keys are raw projections, rotated here at their positions 0 .. s-1; with ``k_rotated`` they
    already hold rope(k) at those positions (a cache that keeps the keys after RoPE) and are used as they
    are.  The query is rotated at its position either way."""
    q_b = as_f64(q_b)
    krows = as_f64(krows)
    vrows = as_f64(vrows)
    h_q, d = q_b.shape
    s, h_kv, _ = krows.shape
    g = h_q // h_kv
    p = s - 1 if include_self else s
    qr = rope(q_b[None, :, :], [p], theta)[0]
    kr = krows if k_rotated else rope(krows, np.arange(s), theta)
    out = np.empty((h_q, d), dtype=np.float64)
    for t in range(h_q):
        u = head_group(t, g)
        a = causal_weights(qr[t][None, :], np.array([p]), kr[:, u, :])
        out[t] = (a @ vrows[:, u, :])[0]
    return out


def packed_offsets(seqlens) -> np.ndarray:
    """off_b = sum of seqlens before b; length B+1 (the packed-cache row index of each sequence)."""
    s = np.asarray(seqlens, dtype=np.int64).reshape(-1)
    return np.concatenate([[0], np.cumsum(s)])


def decode_ref(q, kcache, vcache, seqlens, theta: float, include_self: bool = False,
               batch_rows=None, k_rotated: bool = False) -> np.ndarray:
    """Decode step over the packed cache.  q [B,h_q,d]; caches [sum(seqlens),h_kv,d] (keys raw, or already
    rotated at their positions with ``k_rotated``, as in decode_one_ref).

    Returns float64 [B,h_q,d], or [len(batch_rows),h_q,d] for a subset of sequences.
    """
    seq = [int(x) for x in (seqlens.tolist() if hasattr(seqlens, "tolist") else seqlens)]
    off = packed_offsets(seq)
    bs = range(len(seq)) if batch_rows is None else list(batch_rows)
    outs = []
    for b in bs:
        o0, o1 = int(off[b]), int(off[b + 1])
        outs.append(decode_one_ref(q[b], kcache[o0:o1], vcache[o0:o1], theta, include_self, k_rotated))
    return np.stack(outs, axis=0)


def decode_paged_ref(q, kpages, vpages, block_table, seqlens, theta: float, batch_rows=None,
                     include_self: bool = False, k_rotated: bool = False) -> np.ndarray:
    """Decode step over a paged cache (nxmr.cn page, §2.4: the cache of each KV head kept in blocks).

    kpages/vpages [num_pages, page_size, h_kv, d]; block_table [B, max_pages]: position j of sequence b is
    slot j % page_size of page block_table[b, j // page_size].  Gathers each sequence's rows in position
    order and applies the decode definition of decode_one_ref (``include_self`` and ``k_rotated`` as there).
    """
    kp, vp, bt = np.asarray(kpages), np.asarray(vpages), np.asarray(block_table)
    page_size = kp.shape[1]
    seq = [int(x) for x in (seqlens.tolist() if hasattr(seqlens, "tolist") else seqlens)]
    bs = range(len(seq)) if batch_rows is None else list(batch_rows)
    outs = []
    for b in bs:
        kr = np.stack([kp[bt[b, j // page_size], j % page_size] for j in range(seq[b])])
        vr = np.stack([vp[bt[b, j // page_size], j % page_size] for j in range(seq[b])])
        outs.append(decode_one_ref(q[b], kr, vr, theta, include_self, k_rotated))
    return np.stack(outs, axis=0)


def qkv_append_ref(x, w_qkv, b_qkv, h_q: int, h_kv: int, d: int, seqlens, kpages, vpages, block_table,
                   rotate_k: bool = False, theta=None):
    """One decode step's projection and cache append (aicoding.csdn.net page, §4.1.3 steps 1-2 and its
    closing paragraph: each step appends the current token's K and V to the cache of the h_kv groups;
    nxmr.cn page, §2.4: that cache kept in pages).

    x [B, d_model] is the new token of each sequence; its projection y = x w_qkv^T + b is split into
    q [B, h_q, d] and the rows k, v [B, h_kv, d].  The token sits at position p_b = seqlens[b] (the cache
    length before the append), so k and v go, un-rotated like every cache row, to slot p_b % page_size of
    page block_table[b, p_b // page_size]; with ``rotate_k`` (a cache that keeps keys after RoPE) k goes
    there as rope(k) at p_b with base ``theta``.  Returns (q float64 [B, h_q, d], un-rotated; the grown key
    and value pages as float64 copies); the inputs are not modified.
    """
    xf, wf = as_f64(x), as_f64(w_qkv)
    y = xf @ wf.T                                         # [B, (h_q + 2 h_kv) d]
    if b_qkv is not None:
        y = y + as_f64(b_qkv)[None, :]
    B = xf.shape[0]
    q = y[:, :h_q * d].reshape(B, h_q, d)
    k = y[:, h_q * d:(h_q + h_kv) * d].reshape(B, h_kv, d)
    v = y[:, (h_q + h_kv) * d:].reshape(B, h_kv, d)
    kp, vp = as_f64(kpages).copy(), as_f64(vpages).copy()
    bt = np.asarray(block_table)
    page_size = kp.shape[1]
    for b in range(B):
        pos = int(np.asarray(seqlens).reshape(-1)[b])
        page = int(bt[b, pos // page_size])
        kp[page, pos % page_size] = rope(k[b][None], [pos], theta)[0] if rotate_k else k[b]
        vp[page, pos % page_size] = v[b]
    return q, kp, vp


def qkv_rope_ref(x, w_qkv, b_qkv, h_q: int, h_kv: int, d: int, theta: float, positions=None):
    """Steps 1-3 of the aicoding.csdn.net page, §4.1.3: projections with bias, split into heads, RoPE.

    x [B, L, d_model]; w_qkv [(h_q + 2 h_kv) d, d_model] holds the rows of W_Q^T, W_K^T, W_V^T (so the
    projection is x @ w_qkv^T, i.e. X W with W = w_qkv^T); b_qkv [(h_q + 2 h_kv) d] or None.  Positions
    are 0 .. L-1 in every batch row (or the given `positions` [L], for checking sampled rows of a longer
    sequence).  Returns float64 arrays in the layouts the CUDA path writes:
    qr [B, h_q, L, d] and kr [B, h_kv, L, d] rotated (head-major), k and v [B, L, h_kv, d] un-rotated
    (token-major: the packed cache rows of the sequence).
    """
    xf, wf = as_f64(x), as_f64(w_qkv)
    B, L, _ = xf.shape
    y = xf @ wf.T                                         # [B, L, (h_q + 2 h_kv) d]
    if b_qkv is not None:
        y = y + as_f64(b_qkv)[None, None, :]
    q = y[..., :h_q * d].reshape(B, L, h_q, d)
    k = y[..., h_q * d:(h_q + h_kv) * d].reshape(B, L, h_kv, d)
    v = y[..., (h_q + h_kv) * d:].reshape(B, L, h_kv, d)
    pos = np.arange(L) if positions is None else np.asarray(positions)
    qr = np.stack([rope(q[b], pos, theta) for b in range(B)]).transpose(0, 2, 1, 3)
    kr = np.stack([rope(k[b], pos, theta) for b in range(B)]).transpose(0, 2, 1, 3)
    return qr, kr, k, v


def out_proj_ref(attn, w_o, residual=None) -> np.ndarray:
    """Steps 5-6 of the aicoding.csdn.net page, §4.1.3: Concat of the heads times W_O, plus the residual.

    attn [T, h_q * d] is the concatenated heads (the prefill output [B, L, h_q, d] viewed as rows);
    w_o [d_model, h_q * d] holds the rows of W_O^T (nn.Linear layout), so AttnOut = attn @ w_o^T;
    residual [T, d_model] (the sub-layer input X_in) or None.  Returns float64 [T, d_model].
    """
    y = as_f64(attn) @ as_f64(w_o).T
    if residual is not None:
        y = y + as_f64(residual)
    return y


def qkv_flops(B: int, L: int, d_model: int, h_q: int, h_kv: int, d: int) -> float:
    """FLOP count of the fused projection: one GEMM of [B*L, d_model] x [d_model, (h_q + 2 h_kv) d]."""
    return 2.0 * B * L * d_model * (h_q + 2 * h_kv) * d


def prefill_flops(B: int, L: int, h_q: int, d: int) -> float:
    """Causal-effective FLOP count: 2 GEMMs x 2 flops x d over the L(L+1)/2 unmasked pairs per head."""
    return 4.0 * B * h_q * d * L * (L + 1) / 2.0


def decode_bytes(seqlens, h_q: int, h_kv: int, d: int, elem: int = 2) -> float:
    """Algorithmic bytes of one decode step: K and V rows read once, plus q read and out written."""
    total = float(np.sum(np.asarray(seqlens, dtype=np.int64)))
    B = len(np.asarray(seqlens).reshape(-1))
    return total * h_kv * d * elem * 2 + 2.0 * B * h_q * d * elem
