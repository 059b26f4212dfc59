"""GPU prefill (libgqa through its C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from grouped_query_attention_gqa_b200 import build
    build.build()
    import grouped_query_attention_gqa_b200 as G
    return G


def run(G, q, k, v, theta):
    dev = torch.device("cuda")
    out = G.prefill(q.to(dev), k.to(dev), v.to(dev), theta=theta)
    assert G.last_error() == 0
    return out.float().cpu().numpy()


SMALL = [
    # (B, L, h_q, h_kv, d)  -- several tiles, ragged tails, GQA / MHA / MQA, both head sizes
    (1, 128, 14, 2, 64),
    (1, 1, 14, 2, 64),
    (2, 5, 4, 2, 128),
    (1, 127, 7, 1, 128),
    (1, 129, 8, 8, 128),
    (2, 300, 14, 2, 64),
    (1, 513, 28, 4, 128),
    (3, 200, 16, 4, 128),
    (1, 1000, 4, 1, 64),
    (1, 300, 32, 2, 128),   # g = 16
    (2, 257, 6, 2, 64),     # g = 3, a ragged last tile
]


@pytest.mark.parametrize("B,L,h_q,h_kv,d", SMALL)
def test_prefill_small_full_output(G, B, L, h_q, h_kv, d):
    w = gi.small("prefill", B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, seed=B * 1000 + L + h_q)
    q, k, v = gi.prefill_inputs(w)
    got = run(G, q, k, v, w.theta)
    ref = R.prefill_ref(q, k, v, w.theta)
    assert_close(got, ref, f"prefill B={B} L={L} h_q={h_q} h_kv={h_kv} d={d}")


def test_prefill_first_row_is_v0_exactly(G):
    w = gi.small("prefill", B=2, L=300, h_q=28, h_kv=4, d=128, seed=5)
    q, k, v = gi.prefill_inputs(w)
    got = run(G, q, k, v, w.theta)
    vv = v.float().numpy()
    for t in range(28):
        assert np.array_equal(got[:, 0, t], vv[:, 0, t // 7])


def test_prefill_gqa_equals_mha_on_expanded_kv(G):
    """The kernel's head->group map against the repeat_interleave expansion, both on the GPU."""
    w = gi.small("prefill", B=1, L=260, h_q=28, h_kv=4, d=128, seed=9)
    q, k, v = gi.prefill_inputs(w)
    a = run(G, q, k, v, w.theta)
    b = run(G, q, k.repeat_interleave(7, dim=2).contiguous(), v.repeat_interleave(7, dim=2).contiguous(),
            w.theta)
    assert np.array_equal(a, b)


def test_prefill_theta_1e4_and_repeat_calls(G):
    w = gi.small("prefill", B=1, L=384, h_q=8, h_kv=2, d=128, seed=11, theta=1.0e4)
    q, k, v = gi.prefill_inputs(w)
    ref = R.prefill_ref(q, k, v, w.theta)
    for _ in range(2):
        assert_close(run(G, q, k, v, w.theta), ref, "theta=1e4")


def spike_inputs(B, L, h_q, h_kv, d, seed, step_log2=9.5, alpha=4.0):
    """Inputs whose running row maximum grows by more than 2^8 from one key tile to the next.

    Q and K are small noise plus a component along the pair of dimensions RoPE turns slowest (d/2-1 and
    d-1; at theta = 1e6 it turns by ~1e-6 rad per position, so the rotation leaves that part of the logits
    unchanged).  Key 128t + 5 of every tile t >= 1 carries a spike whose logit is step_log2 * t in log2
    units; all other logits stay near 0.  A row of query tile 1 thus weighs its 128 + 127 plain keys
    against one spike ~2^9.5 times heavier: the lazy rescale of the running output has to happen, and the
    plain keys still make ~15 % of the result, so a wrong rescale shows.
    """
    gen = torch.Generator().manual_seed(seed)
    q = 0.3 * torch.randn(B, L, h_q, d, generator=gen)
    k = 0.3 * torch.randn(B, L, h_kv, d, generator=gen)
    v = torch.randn(B, L, h_kv, d, generator=gen)
    slow = [d // 2 - 1, d - 1]
    q[..., slow] += alpha
    beta = step_log2 * np.log(2.0) * np.sqrt(d) / (2 * alpha)   # spike component per tile step
    for t in range(1, (L + 127) // 128):
        if 128 * t + 5 < L:
            k[:, 128 * t + 5, :, slow] += beta * t
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


@pytest.mark.parametrize("B,L,h_q,h_kv,d", [(1, 700, 28, 4, 128), (2, 400, 8, 2, 64)])
def test_prefill_running_max_grows_across_key_tiles(G, B, L, h_q, h_kv, d):
    q, k, v = spike_inputs(B, L, h_q, h_kv, d, seed=L + d)
    # The construction does what it says: unrotated logits (the rotation moves them by < 1e-3 here) of the
    # spikes step up by more than 8 log2 units per key tile.
    qf, kf = q.float().numpy(), k.float().numpy()
    lg = np.einsum("d,d->", qf[0, L - 1, 0], kf[0, 128 + 5, 0]) / np.sqrt(d) / np.log(2.0)
    lg2 = np.einsum("d,d->", qf[0, L - 1, 0], kf[0, 256 + 5, 0]) / np.sqrt(d) / np.log(2.0)
    assert lg > 8.5 and lg2 - lg > 8.5
    got = run(G, q, k, v, 1.0e6)
    ref = R.prefill_ref(q, k, v, 1.0e6)
    assert_close(got, ref, f"spiked prefill B={B} L={L} d={d}")


def sample_rows(L, rng, n=24):
    fixed = {0, 1, 127, 128, 129, 255, 256, L // 2, L - 2, L - 1}
    rows = {r for r in fixed if 0 <= r < L} | set(rng.integers(0, L, n).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", ["qwen2-0.5b-prefill-L128", "qwen2-7b-prefill-L4096",
                                  "qwen2-72b-prefill-B4-L8192", "qwen2-7b-prefill-L32768"])
def test_prefill_full_size_sampled_rows(G, name):
    """Full workload sizes, same launch as the benchmark; the oracle checks sampled rows."""
    w = gi.BY_NAME[name]
    q, k, v = gi.prefill_inputs(w)
    dev = torch.device("cuda")
    out = G.prefill(q.to(dev), k.to(dev), v.to(dev), theta=w.theta)
    assert G.last_error() == 0
    rng = np.random.default_rng(w.seed)
    heads = sorted({0, w.h_q - 1, w.g, *rng.integers(0, w.h_q, 3).tolist()})
    vv = v[:, 0].float().numpy()
    row0 = out[:, 0].float().cpu().numpy()
    for t in range(w.h_q):   # row 0 of every head is v_0 of its group, exactly
        assert np.array_equal(row0[:, t], vv[:, t // w.g])
    for b in sorted({0, w.B - 1}):
        for t in heads:
            rows = sample_rows(w.L, rng)
            got = out[b, torch.as_tensor(rows, device=dev), t].float().cpu().numpy()
            ref = R.prefill_rows_ref(q, k, v, w.theta, b, t, rows)
            assert_close(got, ref, f"{name} b={b} t={t}")


@pytest.mark.parametrize("B,L,h_q,h_kv,d,expect_grouped", [
    (2, 4096, 28, 4, 128, False),   # many items per CTA, every plane's K' and V in L2: the round-robin lists
    (4, 2048, 14, 2, 64, False),    # the same with d = 64
    (16, 2048, 28, 4, 128, True),   # 64 planes of 1 MB: 64 MB of K' and V, dealt plane group by plane group
])
def test_prefill_schedule_paths_sampled_rows(G, B, L, h_q, h_kv, d, expect_grouped):
    """The attention kernel's other work schedules, checked on sampled rows of the first, a middle and the
    last batch row and of the first, a middle and the last head."""
    lists, grouped = G.prefill_schedule(B, L, h_q, h_kv, 148)
    assert grouped == expect_grouped
    w = gi.small("prefill", B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, seed=B * 100 + L)
    q, k, v = gi.prefill_inputs(w)
    dev = torch.device("cuda")
    out = G.prefill(q.to(dev), k.to(dev), v.to(dev), theta=w.theta)
    assert G.last_error() == 0
    rng = np.random.default_rng(B + L)
    for b in sorted({0, B // 2, B - 1}):
        for t in sorted({0, h_q // 2, h_q - 1}):
            rows = sample_rows(L, rng)
            got = out[b, torch.as_tensor(rows, device=dev), t].float().cpu().numpy()
            ref = R.prefill_rows_ref(q, k, v, w.theta, b, t, rows)
            assert_close(got, ref, f"B={B} L={L} b={b} t={t}")
