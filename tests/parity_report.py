"""Print the parity of the CUDA path against the fp64 oracle for the five workloads (needs a GPU).

    python tests/parity_report.py

Small workload: full output.  Large prefill workloads: every head's row 0 and sampled rows of a few
heads (the oracle computes them one by one).  Decode: six sampled sequences, shortest and longest
included.  Prints max / mean absolute error per workload.  Not collected by pytest (the pass/fail
checks live in test_parity_*.py); this is the table the documentation quotes.
"""
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import gqa_inputs as gi  # noqa: E402
import grouped_query_attention_gqa_b200 as G  # noqa: E402
from oracle import gqa_ref as R  # noqa: E402


def main():
    dev = torch.device("cuda")
    rows = []
    for w in gi.WORKLOADS:
        if w.kind == "prefill":
            q, k, v = gi.prefill_inputs(w)
            out = G.prefill(q.to(dev), k.to(dev), v.to(dev), theta=w.theta)
            assert G.last_error() == 0
            if w.L * w.B <= 4096 and w.h_q <= 28 and w.L <= 512:
                got = out.float().cpu().numpy()
                ref = R.prefill_ref(q, k, v, w.theta)
                what = "full output"
            else:
                rng = np.random.default_rng(w.seed)
                got, ref = [], []
                for b in sorted({0, w.B - 1}):
                    for t in sorted({0, w.g, w.h_q - 1}):
                        rs = np.array(sorted({0, 1, 127, 128, w.L // 2, w.L - 1} | set(rng.integers(0, w.L, 12).tolist())))
                        got.append(out[b, torch.as_tensor(rs, device=dev), t].float().cpu().numpy())
                        ref.append(R.prefill_rows_ref(q, k, v, w.theta, b, t, rs))
                got, ref = np.concatenate(got), np.concatenate(ref)
                what = f"{got.shape[0]} sampled rows"
        else:
            s, q, kc, vc = gi.decode_inputs(w)
            out = G.decode(q.to(dev), kc.to(dev), vc.to(dev), s.to(dev), theta=w.theta)
            assert G.last_error() == 0
            lens = s.numpy()
            pick = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, w.B - 1, 17, 42})
            got = out.float().cpu().numpy()[pick]
            ref = R.decode_ref(q, kc, vc, s, w.theta, batch_rows=pick)
            what = f"{len(pick)} sampled sequences"
        d = np.abs(np.asarray(got, dtype=np.float64) - ref)
        rows.append({"workload": w.name, "checked": what, "max_abs_err": float(d.max()), "mean_abs_err": float(d.mean())})
        print(json.dumps(rows[-1]), flush=True)


if __name__ == "__main__":
    main()
