"""Writes tests/golden/tiny_oracle.json from the oracle alone.

Workload: the tiny case (2 groups x 4 responses, lengths U{16..64}, d=256, V=4096,
H ~ N(0,1), W ~ N(0,1/d) in bf16, uniform token ids, Bernoulli(0.3) rewards,
lp_rollout = oracle lp + N(0, 0.05)), seed 101.  The values are a regression record of
the fp64 oracle; nothing here comes from the CUDA library.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads as wl  # noqa: E402


def compute():
    p = wl.tiny()
    lp, _ = oracle.token_logprobs(p.H, p.W, p.ids)
    lr = wl.rollout_logprobs_with_lag(lp, p.noise, p.seed)
    out = oracle.loss_fwd_bwd(p.H, p.W, p.ids, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids,
                              p.seg.n_groups)
    return dict(
        workload="tiny", seed=p.seed, n_tok=p.n_tok, d=p.d, V=p.V,
        loss=out["loss"],
        lp_first16=[float(x) for x in out["lp"][:16]],
        lse_mean=float(out["lse"].mean()),
        kappa_sum=float(out["kappa"].sum()),
        dH_fro=float(np.linalg.norm(out["dH"])),
        dW_fro=float(np.linalg.norm(out["dW"])),
        dW_row0_first4=[float(x) for x in out["dW"][0, :4]],
    )


if __name__ == "__main__":
    rec = compute()
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json"), "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec)[:200])
