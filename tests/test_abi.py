"""The C-ABI library loads and exports every symbol include/rz.h declares, and its
host-side logic (workspace queries, argument checks) behaves as documented.  CPU only:
no call here reaches the GPU (every call returns before its first CUDA API call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rz.h")


@pytest.fixture(scope="module")
def rz():
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    import invariant_logprobs_reinforce_b200 as rz
    return rz


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rz_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("rz_token_logprobs", "rz_loss_fwd_bwd", "rz_workspace_bytes_logprobs",
                     "rz_workspace_bytes_loss", "rz_read_device_status", "rz_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(rz):
    lib = ctypes.CDLL(rz.build.LIB)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(rz.EXPORTED_SYMBOLS)


def test_status_strings(rz):
    for code, name in rz.STATUS_NAMES.items():
        assert rz.rz_status_string(code) == name
    assert rz.rz_status_string(99) == "RZ_UNKNOWN_STATUS"


def test_workspace_queries(rz):
    assert rz.rz_workspace_bytes_logprobs(1000, 256, 4096) > 0
    assert rz.rz_workspace_bytes_logprobs(0, 256, 4096) > 0
    assert rz.rz_workspace_bytes_logprobs(10, 100, 4096) == 0  # d not a multiple of 64
    assert rz.rz_workspace_bytes_logprobs(10, 256, 0) == 0
    a = rz.rz_workspace_bytes_logprobs(1 << 20, 2560, 151936)
    # (2 * segments + 1) fp32 per token: 75 segments of 2048 columns at V = 151936
    assert a >= (2 * 75 + 1) * 4 * (1 << 20)
    b = rz.rz_workspace_bytes_loss(1 << 20, 512, 64, 2560, 151936)
    # one 16-bit chunk of 16384 x V for the exponentials / dZ, per-chunk partials and tile
    # maxima, and lp, lse, kappa for every token
    assert b >= 16384 * 151936 * 2 + 16384 * 594 * 4 + (2 * 75 + 1) * 4 * 16384 + 12 * (1 << 20)
    assert b < 16384 * 151936 * 2 + 16384 * 594 * 4 + (2 * 75 + 1) * 4 * 16384 + 40 * (1 << 20)
    assert rz.rz_workspace_bytes_loss(0, 1, 1, 256, 4096) == 0
    assert rz.rz_workspace_bytes_segment_loss(100, 4, 2) > 0


def _call_logprobs(lib, H=256, W=512, ids=1024, n=100, d=256, V=4096, lp=2048, lse=None, ws=4096, ws_bytes=None):
    wsb = ws_bytes if ws_bytes is not None else (1 << 40)
    return lib.rz_token_logprobs(H, W, ids, n, d, V, lp, lse, ws, wsb, None)


def test_host_argument_checks_logprobs(rz):
    lib = rz.lib()
    assert _call_logprobs(lib, n=0, H=None, W=None, ids=None, lp=None, ws=None) == 0  # empty call: no-op
    assert _call_logprobs(lib, d=100) == 2
    assert _call_logprobs(lib, d=32) == 2
    assert _call_logprobs(lib, V=0) == 2
    assert _call_logprobs(lib, n=-1) == 1
    assert _call_logprobs(lib, H=None) == 1
    assert _call_logprobs(lib, lp=None) == 1
    assert _call_logprobs(lib, ws=None) == 1
    assert _call_logprobs(lib, H=258) == 1  # H not 16-byte aligned
    assert _call_logprobs(lib, ws=4096 + 16) == 1  # workspace not 256-byte aligned
    assert _call_logprobs(lib, ws_bytes=1024) == 3


def test_host_argument_checks_loss(rz):
    lib = rz.lib()

    def call(**kw):
        a = dict(H=256, W=512, ids=1024, lr=2048, r=3072, off=4096, gid=5120, n=100, R=4, G=2, d=256, V=4096,
                 loss=6144, dH=7168, dW=8192, lp=None, kappa=None, ws=1 << 20, wsb=1 << 40)
        a.update(kw)
        return lib.rz_loss_fwd_bwd(a["H"], a["W"], a["ids"], a["lr"], a["r"], a["off"], a["gid"], a["n"], a["R"],
                                   a["G"], a["d"], a["V"], a["loss"], a["dH"], a["dW"], a["lp"], a["kappa"], a["ws"],
                                   a["wsb"], None)

    assert call(n=0) == 1
    assert call(R=0) == 1
    assert call(G=0) == 1
    assert call(d=96) == 2
    assert call(dW=None) == 1
    assert call(off=4100) == 1  # int64 offsets not 8-byte aligned
    assert call(dH=7170) == 1
    assert call(wsb=100) == 3
    lib2 = rz.lib()
    assert lib2.rz_segment_loss(256, 512, 768, 1024, 1280, 10, 0, 1, 1536, 1792, None, 1 << 20, 1 << 40, None) == 1
    assert lib2.rz_segment_loss(256, 512, 768, 1024, 1280, 10, 2, 1, 1536, 1792, None, 1 << 20, 10, None) == 3


def test_binding_fails_loudly_without_the_native_library():
    """No fallback: with librz.so missing, the first call raises instead of computing."""
    import subprocess
    import sys
    code = (
        "import invariant_logprobs_reinforce_b200 as rz\n"
        "rz._LIB_PATH = '/nonexistent/librz.so'\n"
        "try:\n"
        "    rz.rz_workspace_bytes_loss(100, 2, 1, 256, 4096)\n"
        "except ImportError as e:\n"
        "    print('raised', e)\n"
    )
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=root, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.startswith("raised") and "not built" in out.stdout


def test_host_argument_checks_streamed(rz):
    lib = rz.lib()

    def call(**kw):
        a = dict(Hh=128, Hd=256, W=512, ids=1024, lr=2048, r=3072, off=4096, gid=5120, n=100, R=4, G=2, d=256,
                 V=4096, loss=6144, dH=7168, dW=8192, ws=1 << 20, wsb=1 << 40)
        a.update(kw)
        return lib.rz_loss_fwd_bwd_streamed(a["Hh"], a["Hd"], a["W"], a["ids"], a["lr"], a["r"], a["off"], a["gid"],
                                            a["n"], a["R"], a["G"], a["d"], a["V"], None, a["loss"], a["dH"],
                                            a["dW"], None, None, a["ws"], a["wsb"], None)

    assert call(Hh=None) == 1   # no host rows
    assert call(Hd=None) == 1   # no device buffer
    assert call(Hd=260) == 1    # device buffer not 16-byte aligned
    assert call(d=96) == 2
    assert call(wsb=100) == 3
