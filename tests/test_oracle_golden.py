"""Oracle regression record, a numpy restatement, thread-count independence (CPU only).

tiny_oracle.json was written by tests/golden/make_golden.py from the oracle alone; the
test guards the oracle against silent drift.  The numpy restatement below is a second,
separately written fp64 version of the same definitions (log-softmax gather, group-mean
advantage, unclipped ratio, per-response token mean, REINFORCE gradient) used as a
cross-check on the tiny workload; the closed-form and invariant pins live in
test_oracle_pins.py.
"""
import json
import os

import numpy as np

import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_oracle.json")


def _numpy_path(H, W, ids, lp_roll, rewards, off, gid, G):
    Z = H @ W.T
    m = Z.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(Z - m).sum(axis=1, keepdims=True)))[:, 0]
    lp = Z[np.arange(len(ids)), ids] - lse
    R = len(rewards)
    means = np.array([rewards[gid == g].mean() if np.any(gid == g) else 0.0 for g in range(G)])
    A = rewards - means[gid]
    L = np.diff(off)
    resp = np.repeat(np.arange(R), L)
    w = np.exp(lp - lp_roll)
    loss = -np.sum(A * np.bincount(resp, weights=w, minlength=R) / L) / R
    kappa = -A[resp] * w / (R * L[resp])
    P = np.exp(Z - lse[:, None])
    onehot = np.zeros_like(P)
    onehot[np.arange(len(ids)), ids] = 1.0
    dZ = kappa[:, None] * (onehot - P)
    return dict(loss=loss, lp=lp, lse=lse, kappa=kappa, dH=dZ @ W, dW=dZ.T @ H)


def _tiny_run(oracle):
    p = wl.tiny()
    lp, _ = oracle.token_logprobs(p.H, p.W, p.ids)
    lr = wl.rollout_logprobs_with_lag(lp, p.noise, p.seed)
    out = oracle.loss_fwd_bwd(p.H, p.W, p.ids, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids,
                              p.seg.n_groups)
    return p, lr, out


def test_golden_record(oracle):
    rec = json.load(open(GOLDEN))
    p, _, out = _tiny_run(oracle)
    assert rec["n_tok"] == p.n_tok and rec["d"] == p.d and rec["V"] == p.V
    assert abs(out["loss"] - rec["loss"]) <= 1e-12 * abs(rec["loss"])
    np.testing.assert_allclose(out["lp"][:16], rec["lp_first16"], rtol=1e-13)
    assert abs(np.linalg.norm(out["dH"]) - rec["dH_fro"]) <= 1e-12 * rec["dH_fro"]
    assert abs(np.linalg.norm(out["dW"]) - rec["dW_fro"]) <= 1e-12 * rec["dW_fro"]
    np.testing.assert_allclose(out["dW"][0, :4], rec["dW_row0_first4"], rtol=1e-11, atol=1e-18)


def test_numpy_restatement_agrees(oracle):
    p, lr, out = _tiny_run(oracle)
    H = wl.bits_to_f32(p.H).astype(np.float64)
    W = wl.bits_to_f32(p.W).astype(np.float64)
    ref = _numpy_path(H, W, p.ids, lr.astype(np.float64), p.seg.rewards.astype(np.float64),
                      p.seg.seg_offsets, p.seg.group_ids, p.seg.n_groups)
    assert abs(out["loss"] - ref["loss"]) <= 1e-12 * max(abs(ref["loss"]), 1e-6)
    np.testing.assert_allclose(out["lp"], ref["lp"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"], ref["lse"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["kappa"], ref["kappa"], rtol=1e-12, atol=1e-18)
    for k in ("dH", "dW"):
        err = np.linalg.norm(out[k] - ref[k]) / np.linalg.norm(ref[k])
        assert err < 1e-12, (k, err)


def test_oracle_results_do_not_depend_on_its_thread_count(tmp_path):
    """The oracle parallelises over independent rows only (no reductions across threads),
    so one thread and all threads give the same bits."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys, numpy as np, oracle, workloads as wl\n"
        "p = wl.tiny()\n"
        "lp, _ = oracle.token_logprobs(p.H, p.W, p.ids)\n"
        "lr = wl.rollout_logprobs_with_lag(lp, p.noise, p.seed)\n"
        "o = oracle.loss_fwd_bwd(p.H, p.W, p.ids, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids,\n"
        "                        p.seg.n_groups)\n"
        "np.savez(sys.argv[1], loss=o['loss'], lp=o['lp'], kappa=o['kappa'], dH=o['dH'], dW=o['dW'],\n"
        "         threads=oracle.num_threads())\n"
    )
    outs = {}
    for threads in ("1", str(max(2, os.cpu_count() or 2))):
        f = str(tmp_path / f"t{threads}.npz")
        env = dict(os.environ, OMP_NUM_THREADS=threads, PYTHONPATH=root)
        r = subprocess.run([sys.executable, "-c", code, f], cwd=root, env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        outs[threads] = np.load(f)
    a, b = outs.values()
    assert int(a["threads"]) == 1 and int(b["threads"]) > 1
    for k in ("loss", "lp", "kappa", "dH", "dW"):
        assert a[k].tobytes() == b[k].tobytes(), k
