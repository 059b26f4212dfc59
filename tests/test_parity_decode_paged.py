"""GPU paged-cache decode (gqa_decode_paged through the C ABI) against the fp64 oracle, and against the
packed-cache decode of the same logical cache, which it must reproduce bit for bit (same slices, same
arithmetic; only where the rows are read from differs)."""
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


def run_paged(G, s, q, kp, vp, table, theta):
    dev = torch.device("cuda")
    out = G.decode_paged(q.to(dev), kp.to(dev), vp.to(dev), table.to(dev), s.to(dev), theta=theta)
    return out, G.last_error()


CASES = [
    # (seqlens, h_q, h_kv, d, page_size)
    ([1, 17, 300], 28, 4, 128, 16),
    ([15, 16, 17, 32, 33], 14, 2, 64, 5),      # page size not a multiple of the 16-row block
    ([1000, 1, 4099], 28, 4, 128, 64),
    ([200, 70], 16, 1, 128, 1),               # one row per page, MQA with two head blocks
    ([5000], 64, 8, 128, 256),                # 72B head shape, one long sequence over many warps
    ([64, 3], 8, 8, 128, 4096),               # pages longer than every sequence, MHA
]


@pytest.mark.parametrize("seqlens,h_q,h_kv,d,page", CASES)
def test_decode_paged_small_full_output(G, seqlens, h_q, h_kv, d, page):
    w = gi.small("decode", B=len(seqlens), max_len=max(seqlens), h_q=h_q, h_kv=h_kv, d=d, seed=sum(seqlens) + page)
    s, q, kp, vp, table, _, kc, vc = gi.decode_paged_inputs(w, page, seqlens=seqlens)
    got, err = run_paged(G, s, q, kp, vp, table, w.theta)
    assert err == 0
    ref = R.decode_paged_ref(q.float().numpy(), kp.float().numpy(), vp.float().numpy(), table.numpy(), s, w.theta)
    assert_close(got.float().cpu().numpy(), ref, f"paged decode {seqlens} page={page}")
    packed = G.decode(q.cuda(), kc.cuda(), vc.cuda(), s.cuda(), theta=w.theta)
    assert torch.equal(got, packed), "paged and packed decode of the same cache differ"


def test_decode_paged_shared_prefix_pages(G):
    """Two sequences whose first pages are the same physical pages (a shared prompt prefix)."""
    w = gi.small("decode", B=3, max_len=100, h_q=28, h_kv=4, d=128, seed=12)
    s, q, kp, vp, table, num_pages, _, _ = gi.decode_paged_inputs(w, 16, seqlens=[80, 100, 40])
    table = table.clone()
    table[1, :3] = table[0, :3]   # rows 0..47 of sequence 1 now read sequence 0's pages
    table[2, :2] = table[0, :2]
    got, err = run_paged(G, s, q, kp, vp, table, w.theta)
    assert err == 0
    ref = R.decode_paged_ref(q.float().numpy(), kp.float().numpy(), vp.float().numpy(), table.numpy(), s, w.theta)
    assert_close(got.float().cpu().numpy(), ref, "shared prefix pages")


def test_decode_paged_bad_entries_are_flagged_and_read_as_zero(G):
    """Entries outside [0, num_pages) and a table too short for its sequence: nothing outside the pages is
    read, the rows concerned count as zero rows, the error word says so, other sequences are exact."""
    w = gi.small("decode", B=4, max_len=64, h_q=8, h_kv=2, d=128, seed=13)
    s, q, kp, vp, table, num_pages, _, _ = gi.decode_paged_inputs(w, 16, seqlens=[40, 33, 64, 20])
    table = table.clone()
    table[0, 1] = -1              # rows 16..31 of sequence 0
    table[1, 2] = num_pages       # row 32 of sequence 1
    good = table.clone()
    got, err = run_paged(G, s, q, kp, vp, table, w.theta)
    assert err & G.DEVERR_PAGE
    out = got.float().cpu().numpy()
    assert np.all(np.isfinite(out))
    ref_ok = R.decode_paged_ref(q.float().numpy(), kp.float().numpy(), vp.float().numpy(), good.numpy(), s, w.theta,
                                batch_rows=[2, 3])
    assert_close(out[[2, 3]], ref_ok, "sequences with valid tables")
    # sequence 0 with rows 16..31 replaced by zero K and V rows
    kz, vz = kp.float().numpy().copy(), vp.float().numpy().copy()
    zero_page = num_pages   # an extra all-zero page for the reference
    kz = np.concatenate([kz, np.zeros_like(kz[:1])])
    vz = np.concatenate([vz, np.zeros_like(vz[:1])])
    tz = good.numpy().copy()
    tz[0, 1] = zero_page
    ref0 = R.decode_paged_ref(q.float().numpy(), kz, vz, tz, s, w.theta, batch_rows=[0])
    assert_close(out[[0]], ref0, "sequence 0 with a missing page read as zeros")
    # the sequence is longer than the table covers: max_pages 2 of 16 rows for a 64-row sequence
    w2 = gi.small("decode", B=1, max_len=64, h_q=8, h_kv=2, d=128, seed=14)
    s2, q2, kp2, vp2, t2, _, _, _ = gi.decode_paged_inputs(w2, 16, seqlens=[64])
    got2, err2 = run_paged(G, s2, q2, kp2, vp2, t2[:, :2].contiguous(), w2.theta)
    assert err2 & G.DEVERR_PAGE
    assert np.all(np.isfinite(got2.float().cpu().numpy()))
    assert G.last_error() == 0


def test_decode_paged_full_size_matches_packed(G):
    """The full Qwen2-7B decode workload (B=64, lengths U[1, 32768]) in 16-row pages: bit-identical to the
    packed decode of the same cache, and the oracle checks a sample of sequences."""
    w = gi.BY_NAME["qwen2-7b-decode-B64"]
    s, q, kp, vp, table, _, kc, vc = gi.decode_paged_inputs(w, 16, device="cuda")
    got, err = run_paged(G, s, q, kp, vp, table, w.theta)
    assert err == 0
    packed = G.decode(q, kc, vc, s, theta=w.theta)
    assert torch.equal(got, packed)
    lens = s.cpu().numpy()
    off = np.concatenate([[0], np.cumsum(lens)])
    pick = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, w.B - 1, 29})
    qh = q[pick].cpu()
    kh = torch.cat([kc[off[b]:off[b + 1]].cpu() for b in pick])
    vh = torch.cat([vc[off[b]:off[b + 1]].cpu() for b in pick])
    ref = R.decode_ref(qh, kh, vh, lens[pick], w.theta)
    assert_close(got[pick].float().cpu().numpy(), ref, "qwen2-7b paged decode B=64 sampled")
