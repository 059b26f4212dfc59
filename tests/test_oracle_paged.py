"""Pins of the paged-cache decode oracle (page "从 Qwen 1 到 Qwen 2", nxmr.cn, §2.4) and of the seeded
paged layout.  The paged decode is defined as the packed decode after reading each position through the
block table, so it is pinned by a brute-force restatement on a hand-made table and by equality with the
(separately pinned) packed oracle on scattered layouts."""
import numpy as np
import pytest
import torch

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.test_oracle_pins import _bf_attend


def _hand_case():
    """page_size 2, sequences of 3 and 4 rows in 5 pages placed out of order (page 4 unused)."""
    rng = np.random.default_rng(11)
    h_q, h_kv, d, P = 4, 2, 8, 2
    kp = rng.standard_normal((5, P, h_kv, d))
    vp = rng.standard_normal((5, P, h_kv, d))
    bt = np.array([[3, 0, -1], [2, 1, -1]], dtype=np.int32)   # seq 0: pages 3,0; seq 1: pages 2,1
    seqlens = [3, 4]
    q = rng.standard_normal((2, h_q, d))
    return q, kp, vp, bt, seqlens, h_q, h_kv, d, P


def _paged_pins_pass(fn):
    q, kp, vp, bt, seqlens, h_q, h_kv, d, P = _hand_case()
    try:
        got = fn(q, kp, vp, bt, seqlens, 10.0)
        for b, s in enumerate(seqlens):
            for t in range(h_q):
                u = t // (h_q // h_kv)
                rows = [(bt[b, j // P], j % P) for j in range(s)]   # position j -> (page, slot)
                ref = _bf_attend(list(q[b, t]), s, [list(kp[pg, sl, u]) for pg, sl in rows],
                                 [list(vp[pg, sl, u]) for pg, sl in rows], 10.0, d)
                if not np.allclose(got[b, t], ref, atol=1e-12):
                    return False
        w = gi.small("decode", B=5, max_len=40, h_q=4, h_kv=2, d=8, seed=9)
        for page in (1, 3, 16):
            s, qq, kpp, vpp, tab, _, kc, vc = gi.decode_paged_inputs(w, page)
            if not np.allclose(fn(qq.float().numpy(), kpp.float().numpy(), vpp.float().numpy(), tab.numpy(), s, w.theta),
                               R.decode_ref(qq.float().numpy(), kc.float().numpy(), vc.float().numpy(), s, w.theta),
                               atol=1e-12):
                return False
        return True
    except Exception:
        return False


def test_paged_ref_matches_brute_force_and_packed():
    assert _paged_pins_pass(R.decode_paged_ref)


def _mut_gather(page_of, slot_of):
    def fn(q, kpages, vpages, block_table, seqlens, theta):
        kp, vp, bt = np.asarray(kpages), np.asarray(vpages), np.asarray(block_table)
        P = kp.shape[1]
        out = []
        for b, s in enumerate(int(x) for x in seqlens):
            idx = [(bt[b, page_of(j, P) % bt.shape[1]], slot_of(j, P) % P) for j in range(s)]
            kr = np.stack([kp[pg, sl] for pg, sl in idx])
            vr = np.stack([vp[pg, sl] for pg, sl in idx])
            out.append(R.decode_one_ref(q[b], kr, vr, theta))
        return np.stack(out)
    return fn


@pytest.mark.parametrize("name,page_of,slot_of", [
    ("page_and_slot_swapped", lambda j, P: j % P, lambda j, P: j // P),
    ("next_page", lambda j, P: j // P + 1, lambda j, P: j % P),
    ("slot_reversed", lambda j, P: j // P, lambda j, P: P - 1 - j % P),
])
def test_paged_pins_catch_planted_mistakes(name, page_of, slot_of):
    assert not _paged_pins_pass(_mut_gather(page_of, slot_of)), name


@pytest.mark.parametrize("page_size", [1, 5, 16, 64, 4096])
def test_paged_layout_is_a_valid_placement(page_size):
    lens = [1, 17, 300, 64, 65]
    table, num_pages, store_row = gi.paged_layout(lens, page_size, seed=3, extra_pages=4)
    need = [(n + page_size - 1) // page_size for n in lens]
    assert num_pages == sum(need) + 4
    assert table.shape == (len(lens), max(need)) and table.dtype == torch.int32
    used = torch.cat([table[b, :need[b]] for b in range(len(lens))])
    assert used.unique().numel() == used.numel() and int(used.min()) >= 0 and int(used.max()) < num_pages
    for b in range(len(lens)):
        assert bool((table[b, need[b]:] == -1).all())
    assert store_row.numel() == sum(lens) and store_row.unique().numel() == sum(lens)
    assert int(store_row.max()) < num_pages * page_size
    # position j of sequence b sits at slot j % page_size of its page
    off = 0
    for b, n in enumerate(lens):
        j = torch.arange(n)
        assert torch.equal(store_row[off:off + n] % page_size, j % page_size)
        assert torch.equal(store_row[off:off + n] // page_size, table[b, j // page_size].long())
        off += n


def test_paged_inputs_scatter_the_packed_rows():
    w = gi.small("decode", B=4, max_len=50, h_q=4, h_kv=2, d=8, seed=5)
    s, q, kp, vp, table, num_pages, kc, vc = gi.decode_paged_inputs(w, 16)
    s2, q2, kc2, vc2 = gi.decode_inputs(w)
    assert torch.equal(s, s2) and torch.equal(q, q2) and torch.equal(kc, kc2) and torch.equal(vc, vc2)
    _, _, store_row = gi.paged_layout(s, 16, w.seed + 7919)
    assert torch.equal(kp.reshape(-1, 2, 8)[store_row], kc) and torch.equal(vp.reshape(-1, 2, 8)[store_row], vc)
