"""Mutation check of the oracle's pins (CPU only).  Each case plants one plausible mistake
in a copy of oracle/oracle.c (every occurrence of the line), rebuilds that copy and runs the
pins against it (tests/test_oracle_pins.py for the method's core, tests/test_oracle_variants.py
for the loss-stage variants and the ratio diagnostics; the e4m3 helpers in oracle/__init__.py
against tests/test_oracle_fp8.py; the MXFP4 reference in oracle/mxfp4.py against
tests/test_oracle_mxfp4.py): some pin must fail.  The unmutated copy is the control for
each pin file and must pass.  Every planted line must still exist
verbatim, so the list cannot silently drift away from the oracle."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "control": None,
    "dropped 1/L_i": ("loss += A[i] * (wsum / L);", "loss += A[i] * wsum;"),
    "dropped 1/N": ("*loss_out = -loss / N;", "*loss_out = -loss;"),
    "flipped loss sign": ("*loss_out = -loss / N;", "*loss_out = loss / N;"),
    "inverted ratio": ("const double w = exp(lp[t] - lp_rollout[t]);",
                       "const double w = exp(lp_rollout[t] - lp[t]);"),
    "global instead of group mean": ("A[i] = rewards[i] - sum[gid[i]] / (double)cnt[gid[i]];",
                                     "A[i] = rewards[i] - sum[0] / (double)cnt[0];"),
    "transposed W index": ("elem(W, (size_t)v * d + k, is_bf16);", "elem(W, (size_t)k * V + v, is_bf16);"),
    "dropped softmax term in dZ": ("(v == ids[t] ? 1.0 : 0.0) - exp(z[v] - lse_rows[j])",
                                   "(v == ids[t] ? 1.0 : 0.0)"),
    "kappa without w": ("if (kappa_out) kappa_out[t] = -A[i] * w / (N * L);",
                        "if (kappa_out) kappa_out[t] = -A[i] / (N * L);"),
    "lp without lse": ("if (lp) lp[j] = z[ids[t]] - l;", "if (lp) lp[j] = z[ids[t]] - z[0];"),
    "wrong dZ sign": ("const double dz = kappa[t] * ((v == ids[t] ? 1.0 : 0.0) - exp(z - lse[t]));",
                      "const double dz = kappa[t] * ((v == ids[t] ? 1.0 : 0.0) + exp(z - lse[t]));"),
}
PINS = "tests/test_oracle_pins.py"

VARIANT_MUTATIONS = {
    "control": None,
    "clip from below": ("if ((flags & ORACLE_CLIP) && w > clip_max) w = clip_max;",
                        "if ((flags & ORACLE_CLIP) && w < clip_max) w = clip_max;"),
    "inverted gate": ("keep = (g >= gate_lo && g <= gate_hi);", "keep = !(g >= gate_lo && g <= gate_hi);"),
    "gate on the summed log-ratio": ("const double g = exp(logsum / L);", "const double g = exp(logsum);"),
    "mask ignored in L_i": ("      if (counted) {\n        L += 1.0;", "      if (1) {\n        L += 1.0;"),
    "global N ignored": ("const double N = n_resp_total > 0 ? (double)n_resp_total : (double)R;",
                         "const double N = (double)R;"),
    "upper median": ("const double med = dev[(m - 1) / 2];", "const double med = dev[m / 2];"),
    "k3 without -x": ("k3 += w - 1.0 - x;", "k3 += w - 1.0;"),
    "k1 sign": ("k1 += -x;", "k1 += x;"),
    "peak over w": ("if (d > dmax) dmax = d;", "if (w > dmax) dmax = w;"),
    "mask ignored in the statistics": ("      if (mask && !mask[t]) continue;\n      const double x = lp[t] - lp_rollout[t];",
                                       "      const double x = lp[t] - lp_rollout[t];"),
}
VARIANT_PINS = "tests/test_oracle_variants.py"

FP8_MUTATIONS = {
    "control": None,
    "e4m3 range of the fnuz variant": ("E4M3_MAX = 448.0", "E4M3_MAX = 240.0"),
    "decoded as e5m2": ("torch.float8_e4m3fn).double()", "torch.float8_e5m2).double()"),
    "no zero-row guard": ("torch.where(m > 0, m / torch.tensor(E4M3_MAX, dtype=torch.float32), torch.ones_like(m))",
                          "m / torch.tensor(E4M3_MAX, dtype=torch.float32)"),
    "scale from the row mean": ("m = x.abs().amax(dim=1)", "m = x.abs().mean(dim=1)"),
    "sign dropped": ("y = (x / sc[:, None])", "y = (x.abs() / sc[:, None])"),
}
FP8_PINS = "tests/test_oracle_fp8.py"

MXFP4_MUTATIONS = {
    "control": None,
    "E2M1 top exponent 1": ("E2M1_EMAX = 2", "E2M1_EMAX = 1"),
    "ceiling block exponent": ("Xe = (e.astype(np.int64) - 1) - E2M1_EMAX", "Xe = e.astype(np.int64) - E2M1_EMAX"),
    "ties to odd": ("even = tie & (np.arange(8) % 2 == 0)", "even = tie & (np.arange(8) % 2 == 1)"),
    "sign dropped": ("return mag | (np.signbit(y).astype(np.uint8) << 3)", "return mag"),
    "E8M0 bias 128": ("return codes, (Xe + 127).astype(np.uint8)", "return codes, (Xe + 128).astype(np.uint8)"),
}
MXFP4_PINS = "tests/test_oracle_mxfp4.py"
TARGETS = {PINS: ("oracle.c", MUTATIONS), VARIANT_PINS: ("oracle.c", VARIANT_MUTATIONS),
           FP8_PINS: ("__init__.py", FP8_MUTATIONS), MXFP4_PINS: ("mxfp4.py", MXFP4_MUTATIONS)}
CASES = [(pins, k) for pins, (_, table) in TARGETS.items() for k in table]


def _copy_tree(dst):
    ignore = shutil.ignore_patterns("*.so", "__pycache__", "*.pyc")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"), ignore=ignore)
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(dst, "tests"), ignore=ignore)
    for f in ("workloads.py", "pytest.ini"):
        shutil.copy(os.path.join(ROOT, f), dst)


def _run_case(root, pins, name):
    """Plant one mistake in a fresh copy under `root` and run its pin file there; returns
    (returncode, stdout, output tail)."""
    _copy_tree(root)
    target, table = TARGETS[pins]
    src_path = os.path.join(root, "oracle", target)
    mutation = table[name]
    if mutation is not None:
        old, new = mutation
        with open(src_path) as f:
            text = f.read()
        if old not in text:
            return None, "", f"planted line no longer in oracle/{target}: {old}"
        with open(src_path, "w") as f:
            f.write(text.replace(old, new))
    # one OpenMP thread per copy: the copies run side by side
    env = dict(os.environ, PYTHONPATH=root, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", pins, "-q", "-x", "-p", "no:cacheprovider"], cwd=root,
                       capture_output=True, text=True, timeout=900, env=env)
    return r.returncode, r.stdout, (r.stdout + r.stderr)[-1500:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Every case, each in its own copy, run concurrently (independent subprocesses)."""
    from concurrent.futures import ThreadPoolExecutor
    roots = {case: str(tmp_path_factory.mktemp("mut")) for case in CASES}
    with ThreadPoolExecutor(max_workers=max(1, min(len(CASES), os.cpu_count() or 1))) as pool:
        futures = {case: pool.submit(_run_case, roots[case], *case) for case in CASES}
        return {case: f.result() for case, f in futures.items()}


@pytest.mark.parametrize("pins,name", CASES)
def test_pins_catch_a_planted_mistake(outcomes, pins, name):
    code, stdout, tail = outcomes[(pins, name)]
    assert code is not None, tail
    if name == "control":
        assert code == 0, tail
    else:
        # 1 = tests ran and some failed (not a build, collection or usage error)
        assert code == 1 and "failed" in stdout, tail
