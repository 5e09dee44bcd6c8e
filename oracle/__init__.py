"""fp64 CPU oracle for the REINFORCE Zero token-logprob / loss / gradient path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` are the only callers.  The product path (the CUDA library and its
binding) never imports this package, and this package imports nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over independent rows); this
module compiles it with gcc and marshals numpy arrays through ctypes.  Each wrapper cites
the page section of "vLLM says aligned kernels make asynchronous RL stable at lag 64"
(ainewsbites.com) that the step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-funswitch-loops", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, c_int = ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        lib.oracle_lp_rows.argtypes = [P, P, c_int, P, i64, i32, i32, P, i64, P, P]
        lib.oracle_advantages.argtypes = [P, P, i32, i32, P]
        lib.oracle_loss_from_lp.argtypes = [P, P, P, P, P, i64, i32, i32, P, P, P]
        lib.oracle_dh_rows.argtypes = [P, P, c_int, P, i64, i32, i32, P, i64, P, P, P]
        lib.oracle_dw_rows.argtypes = [P, P, c_int, P, i64, i32, i32, P, P, P, i64, P]
        lib.oracle_loss_fwd_bwd.argtypes = [P, P, c_int, P, P, P, P, P, i64, i32, i32, i32, i32,
                                            P, P, P, P, P, P, P]
        lib.oracle_num_threads.argtypes = []
        lib.oracle_loss_from_lp_ex.argtypes = [P, P, P, P, P, i64, i32, i32, i32, ctypes.c_double, ctypes.c_double,
                                               ctypes.c_double, P, i32, P, P, P]
        lib.oracle_ratio_stats.argtypes = [P, P, P, i64, i32, P, P, P]
        for f in ("oracle_lp_rows", "oracle_advantages", "oracle_loss_from_lp", "oracle_dh_rows",
                  "oracle_dw_rows", "oracle_loss_fwd_bwd", "oracle_num_threads", "oracle_loss_from_lp_ex",
                  "oracle_ratio_stats"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _mat(x):
    """Matrix operand: uint16 arrays are bf16 bit patterns, anything else is taken as fp64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), 1
    return np.ascontiguousarray(x, dtype=np.float64), 0


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle returned {rc} ({'invalid argument' if rc == 1 else 'out of memory'})")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def token_logprobs(H, W, ids, rows=None):
    """lp and lse of the listed rows (all rows if ``rows`` is None).

    The learner's own log-probability of each sampled token: log-softmax of the LM-head
    logits z = H W^T gathered at the token ("REINFORCE Zero removes the mismatch first").
    Returns (lp, lse), fp64.
    """
    lib = _load()
    Hm, bf = _mat(H)
    Wm, bf2 = _mat(W)
    assert bf == bf2, "H and W must both be bf16 bits or both be float"
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n, d = Hm.shape
    V = Wm.shape[0]
    assert Wm.shape[1] == d and ids.shape == (n,)
    if rows is None:
        r, nrows = None, n
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = r.shape[0]
    lp = np.empty(nrows, np.float64)
    lse = np.empty(nrows, np.float64)
    _check(lib.oracle_lp_rows(_ptr(Hm), _ptr(Wm), bf, _ptr(ids), n, d, V, _ptr(r), nrows, _ptr(lp),
                              _ptr(lse)), "token_logprobs")
    return lp, lse


def advantages(rewards, group_ids, n_groups):
    """A_i = r_i - mean reward of response i's group (group mean includes response i)."""
    lib = _load()
    r = np.ascontiguousarray(rewards, dtype=np.float64)
    g = np.ascontiguousarray(group_ids, dtype=np.int32)
    A = np.empty(r.shape[0], np.float64)
    _check(lib.oracle_advantages(_ptr(r), _ptr(g), r.shape[0], n_groups, _ptr(A)), "advantages")
    return A


def loss_from_lp(lp, lp_rollout, rewards, seg_offsets, group_ids, n_groups):
    """(loss, w, kappa) from per-token logprobs.

    w_t = exp(lp_t - lp_rollout_t), unclipped; loss = -(1/N) sum_i A_i mean_{t in i} w_t;
    kappa_t = d loss / d lp_t = -A_i w_t / (N L_i).
    """
    lib = _load()
    lp = np.ascontiguousarray(lp, dtype=np.float64)
    lr = np.ascontiguousarray(lp_rollout, dtype=np.float64)
    r = np.ascontiguousarray(rewards, dtype=np.float64)
    off = np.ascontiguousarray(seg_offsets, dtype=np.int64)
    g = np.ascontiguousarray(group_ids, dtype=np.int32)
    n, R = lp.shape[0], r.shape[0]
    w = np.empty(n, np.float64)
    kappa = np.empty(n, np.float64)
    loss = np.zeros(1, np.float64)
    _check(lib.oracle_loss_from_lp(_ptr(lp), _ptr(lr), _ptr(r), _ptr(off), _ptr(g), n, R, n_groups,
                                   _ptr(w), _ptr(kappa), _ptr(loss)), "loss_from_lp")
    return float(loss[0]), w, kappa


def dh_rows(H, W, ids, rows, lse_rows, kappa_rows):
    """dH of the listed rows given their lse and kappa: sum_v kappa([v=y]-p_v) W[v,:]."""
    lib = _load()
    Hm, bf = _mat(H)
    Wm, _ = _mat(W)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n, d = Hm.shape
    V = Wm.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = n if r is None else r.shape[0]
    ls = np.ascontiguousarray(lse_rows, dtype=np.float64)
    ka = np.ascontiguousarray(kappa_rows, dtype=np.float64)
    out = np.empty((nrows, d), np.float64)
    _check(lib.oracle_dh_rows(_ptr(Hm), _ptr(Wm), bf, _ptr(ids), n, d, V, _ptr(r), nrows, _ptr(ls),
                              _ptr(ka), _ptr(out)), "dh_rows")
    return out


def dw_rows(H, W, ids, lse, kappa, vocab_rows=None):
    """dW of the listed vocabulary rows: sum_t kappa_t([v=y_t]-p_tv) H[t,:]."""
    lib = _load()
    Hm, bf = _mat(H)
    Wm, _ = _mat(W)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n, d = Hm.shape
    V = Wm.shape[0]
    vr = None if vocab_rows is None else np.ascontiguousarray(vocab_rows, dtype=np.int64)
    nv = V if vr is None else vr.shape[0]
    ls = np.ascontiguousarray(lse, dtype=np.float64)
    ka = np.ascontiguousarray(kappa, dtype=np.float64)
    out = np.empty((nv, d), np.float64)
    _check(lib.oracle_dw_rows(_ptr(Hm), _ptr(Wm), bf, _ptr(ids), n, d, V, _ptr(ls), _ptr(ka), _ptr(vr),
                              nv, _ptr(out)), "dw_rows")
    return out


def loss_fwd_bwd(H, W, ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups,
                 want_dh=True, want_dw=True):
    """The whole path in fp64.  Returns a dict with loss, lp, lse, w, kappa, dH, dW."""
    lib = _load()
    Hm, bf = _mat(H)
    Wm, bf2 = _mat(W)
    assert bf == bf2
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n, d = Hm.shape
    V = Wm.shape[0]
    lr = np.ascontiguousarray(lp_rollout, dtype=np.float64)
    r = np.ascontiguousarray(rewards, dtype=np.float64)
    off = np.ascontiguousarray(seg_offsets, dtype=np.int64)
    g = np.ascontiguousarray(group_ids, dtype=np.int32)
    R = r.shape[0]
    loss = np.zeros(1, np.float64)
    dH = np.empty((n, d), np.float64) if want_dh else None
    dW = np.empty((V, d), np.float64) if want_dw else None
    lp = np.empty(n, np.float64)
    lse = np.empty(n, np.float64)
    w = np.empty(n, np.float64)
    kappa = np.empty(n, np.float64)
    _check(lib.oracle_loss_fwd_bwd(_ptr(Hm), _ptr(Wm), bf, _ptr(ids), _ptr(lr), _ptr(r), _ptr(off),
                                   _ptr(g), n, R, n_groups, d, V, _ptr(loss), _ptr(dH), _ptr(dW),
                                   _ptr(lp), _ptr(lse), _ptr(w), _ptr(kappa)), "loss_fwd_bwd")
    return dict(loss=float(loss[0]), lp=lp, lse=lse, w=w, kappa=kappa, dH=dH, dW=dW)


CLIP, GATE, MASK = 1, 2, 4


def loss_from_lp_ex(lp, lp_rollout, rewards, seg_offsets, group_ids, n_groups, flags=0, clip_max=float("inf"),
                    gate_lo=0.0, gate_hi=float("inf"), mask=None, n_resp_total=0):
    """(loss, w, kappa) of the loss-stage variants (truncated IS, sequence gate, token mask,
    global response count); flags = 0 reproduces loss_from_lp.  Readings in oracle.c."""
    lib = _load()
    lp = np.ascontiguousarray(lp, dtype=np.float64)
    lr = np.ascontiguousarray(lp_rollout, dtype=np.float64)
    r = np.ascontiguousarray(rewards, dtype=np.float64)
    off = np.ascontiguousarray(seg_offsets, dtype=np.int64)
    g = np.ascontiguousarray(group_ids, dtype=np.int32)
    mk = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    n, R = lp.shape[0], r.shape[0]
    w = np.empty(n, np.float64)
    kappa = np.empty(n, np.float64)
    loss = np.zeros(1, np.float64)
    _check(lib.oracle_loss_from_lp_ex(_ptr(lp), _ptr(lr), _ptr(r), _ptr(off), _ptr(g), n, R, n_groups, flags,
                                      clip_max, gate_lo, gate_hi, _ptr(mk), n_resp_total, _ptr(w), _ptr(kappa),
                                      _ptr(loss)), "loss_from_lp_ex")
    return float(loss[0]), w, kappa


STAT_NAMES = ("k1", "k2", "k3", "w_min", "w_max", "dev_max", "dev_median", "dev_peak_over_median", "count")


def ratio_stats(lp, lp_rollout, seg_offsets, mask=None):
    """Ratio diagnostics (dict keyed by STAT_NAMES) and the per-response mean ratio."""
    lib = _load()
    lp = np.ascontiguousarray(lp, dtype=np.float64)
    lr = np.ascontiguousarray(lp_rollout, dtype=np.float64)
    off = np.ascontiguousarray(seg_offsets, dtype=np.int64)
    mk = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    n, R = lp.shape[0], off.shape[0] - 1
    stats = np.empty(9, np.float64)
    rm = np.empty(R, np.float64)
    _check(lib.oracle_ratio_stats(_ptr(lp), _ptr(lr), _ptr(off), n, R, _ptr(mk), _ptr(stats), _ptr(rm)),
           "ratio_stats")
    return dict(zip(STAT_NAMES, stats.tolist())), rm


E4M3_MAX = 448.0


def quantize_rows_e4m3(X_bits):
    """Per-row e4m3 codes of a bf16 matrix (uint16 bit patterns): scale = max|x| / 448 in fp32
    (1 for an all-zero row), code = e4m3(x / scale) with fp32 division, round to nearest
    even (torch's CPU conversion).  Returns (codes uint8 [rows, d], scale fp32 [rows])."""
    import torch
    x = torch.from_numpy(np.ascontiguousarray(X_bits).view(np.int16)).view(torch.bfloat16).float()
    m = x.abs().amax(dim=1)
    sc = torch.where(m > 0, m / torch.tensor(E4M3_MAX, dtype=torch.float32), torch.ones_like(m))
    y = (x / sc[:, None]).clamp(-E4M3_MAX, E4M3_MAX)
    q = y.to(torch.float8_e4m3fn)
    return q.view(torch.uint8).numpy().copy(), sc.numpy().copy()


def decode_e4m3(codes):
    """fp64 values of e4m3 codes (uint8)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
