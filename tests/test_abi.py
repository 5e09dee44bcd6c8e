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

    def host_io(**kw):
        a = dict(Hh=128, Hd=256, W=512, ids=1024, lr=2048, r=3072, off=4096, gid=5120, n=100, R=4, G=2, d=256,
                 V=4096, loss=6144, dH=7168, dW=8192, dHh=9216, dWh=10240, ws=1 << 20, wsb=1 << 40)
        a.update(kw)
        return lib.rz_loss_fwd_bwd_host_io(a["Hh"], a["Hd"], a["W"], a["ids"], a["lr"], a["r"], a["off"], a["gid"],
                                           a["n"], a["R"], a["G"], a["d"], a["V"], None, a["loss"], a["dH"],
                                           a["dW"], None, None, a["dHh"], a["dWh"], a["ws"], a["wsb"], None)

    assert host_io(Hh=None) == 1 and host_io(Hd=None) == 1 and host_io(d=96) == 2 and host_io(wsb=100) == 3
    assert host_io(n=0) == 1


def _opts(rz, **kw):
    o = rz.rz_loss_options()
    o.flags, o.clip_max, o.gate_lo, o.gate_hi, o.token_mask, o.n_resp_total = 0, 0.0, 0.0, 0.0, None, 0
    for k, v in kw.items():
        setattr(o, k, v)
    return o


def _bad_options(rz):
    C, G, M = rz.RZ_LOSS_CLIP_IS, rz.RZ_LOSS_SEQ_GATE, rz.RZ_LOSS_TOKEN_MASK
    return [
        _opts(rz, flags=8),                              # unknown flag bit
        _opts(rz, flags=C, clip_max=0.0),                # clip_max must be > 0
        _opts(rz, flags=C, clip_max=float("nan")),
        _opts(rz, flags=G, gate_lo=2.0, gate_hi=1.0),    # empty gate interval
        _opts(rz, flags=M, token_mask=None),             # mask flag without a mask
        _opts(rz, flags=M, token_mask=4098),             # mask not 4-byte aligned
        _opts(rz, n_resp_total=-1),
    ]


def test_host_checks_of_the_loss_options(rz):
    import ctypes
    lib = rz.lib()

    def ex(opt, d=256, wsb=1 << 40):
        return lib.rz_loss_fwd_bwd_ex(256, 512, 1024, 2048, 3072, 4096, 5120, 100, 4, 2, d, 4096,
                                      ctypes.byref(opt), 6144, 7168, 8192, None, None, 1 << 20, wsb, None)

    def seg_ex(opt, wsb=1 << 40):
        return lib.rz_segment_loss_ex(256, 512, 768, 1024, 1280, 10, 2, 1, ctypes.byref(opt), 1536, 1792, None,
                                      1 << 20, wsb, None)

    for o in _bad_options(rz):
        assert ex(o) == 1 and seg_ex(o) == 1
        assert ex(o, d=96) == 1  # the options are checked before the shape
    good = _opts(rz, flags=rz.RZ_LOSS_CLIP_IS | rz.RZ_LOSS_SEQ_GATE | rz.RZ_LOSS_TOKEN_MASK, clip_max=2.0,
                 gate_lo=0.5, gate_hi=2.0, token_mask=4096, n_resp_total=7)
    assert ex(good, d=96) == 2
    assert ex(good, wsb=100) == 3 and seg_ex(good, wsb=10) == 3


def test_host_checks_of_the_diagnostics(rz):
    lib = rz.lib()
    assert rz.rz_workspace_bytes_ratio_stats(0, 1) == 0 and rz.rz_workspace_bytes_ratio_stats(10, 0) == 0
    assert rz.rz_workspace_bytes_ratio_stats(1 << 20, 100) > 0
    assert rz.rz_workspace_bytes_grad_norms() >= 2 * 8 * 148

    def stats(**kw):
        a = dict(lp=256, lr=512, off=768, n=100, R=3, mask=None, out=1024, rm=None, ws=1 << 20, wsb=1 << 40)
        a.update(kw)
        return lib.rz_ratio_stats(a["lp"], a["lr"], a["off"], a["n"], a["R"], a["mask"], a["out"], a["rm"],
                                  a["ws"], a["wsb"], None)

    assert stats(n=0) == 1 and stats(R=0) == 1 and stats(lp=None) == 1 and stats(out=None) == 1
    assert stats(off=772) == 1   # int64 offsets not 8-byte aligned
    assert stats(out=1028) == 1  # fp64 outputs not 8-byte aligned
    assert stats(rm=1026) == 1 and stats(ws=(1 << 20) + 64) == 1
    assert stats(wsb=100) == 3

    def norms(**kw):
        a = dict(dH=256, dW=512, n=10, d=64, V=100, out=1024, ws=1 << 20, wsb=1 << 40)
        a.update(kw)
        return lib.rz_grad_norms(a["dH"], a["dW"], a["n"], a["d"], a["V"], a["out"], a["ws"], a["wsb"], None)

    assert norms(n=-1) == 1 and norms(d=0) == 1 and norms(V=-1) == 1 and norms(out=None) == 1
    assert norms(dH=None) == 1 and norms(dW=None) == 1 and norms(out=1028) == 1
    assert norms(wsb=8) == 3


def test_host_checks_of_the_fp8_forward(rz):
    lib = rz.lib()
    assert lib.rz_quantize_rows_e4m3(256, -1, 64, 512, 1024, None) == 1
    assert lib.rz_quantize_rows_e4m3(256, 10, 0, 512, 1024, None) == 1
    assert lib.rz_quantize_rows_e4m3(None, 0, 64, None, None, None) == 0   # no rows: a no-op
    assert lib.rz_quantize_rows_e4m3(None, 10, 64, 512, 1024, None) == 1
    assert lib.rz_quantize_rows_e4m3(256, 10, 64, 512, 1026, None) == 1    # scales not 4-byte aligned

    def fwd(**kw):
        a = dict(H=256, hs=512, W=1024, ws_=2048, ids=3072, n=100, d=256, V=4096, lp=4096 + 256, lse=None,
                 ws=1 << 20, wsb=1 << 40)
        a.update(kw)
        return lib.rz_token_logprobs_fp8(a["H"], a["hs"], a["W"], a["ws_"], a["ids"], a["n"], a["d"], a["V"], a["lp"],
                                         a["lse"], a["ws"], a["wsb"], None)

    assert fwd(d=192) == 2 and fwd(d=100) == 2 and fwd(V=0) == 2  # d a multiple of 128
    assert fwd(n=-1) == 1
    assert fwd(n=0, H=None, hs=None, W=None, ws_=None, ids=None, lp=None, ws=None) == 0
    assert fwd(H=None) == 1 and fwd(hs=None) == 1 and fwd(H=264) == 1 and fwd(ws_=2050) == 1
    assert fwd(wsb=100) == 3


def test_host_checks_of_the_shard_sum_selftest_noalloc_and_timed(rz):
    import ctypes
    lib = rz.lib()
    assert lib.rz_sum_shards_f32(256, 0, 10, 512, None) == 1
    assert lib.rz_sum_shards_f32(256, 2, -1, 512, None) == 1
    assert lib.rz_sum_shards_f32(None, 2, 0, None, None) == 0   # nothing to sum
    assert lib.rz_sum_shards_f32(None, 2, 10, 512, None) == 1
    assert lib.rz_sum_shards_f32(256, 2, 10, 514, None) == 1

    waited = ctypes.c_uint64(0)
    assert lib.rz_selftest_wait_timeout(1000, None, 256, ctypes.byref(waited), None) == 1
    assert lib.rz_selftest_wait_timeout(1000, 1 << 20, 100, ctypes.byref(waited), None) == 1
    assert lib.rz_selftest_wait_timeout(10_000_000_001, 1 << 20, 256, ctypes.byref(waited), None) == 1
    assert lib.rz_selftest_wait_timeout(1000, (1 << 20) + 16, 256, ctypes.byref(waited), None) == 1

    def noalloc(**kw):
        a = dict(H=256, W=512, ids=1024, n=100, d=256, V=4096, lp=2048, lse=None)
        a.update(kw)
        return lib.rz_token_logprobs_noalloc(a["H"], a["W"], a["ids"], a["n"], a["d"], a["V"], a["lp"], a["lse"],
                                             None)

    assert noalloc(n=-1) == 1 and noalloc(d=96) == 2
    assert noalloc(n=0, H=None, W=None, ids=None, lp=None) == 0
    assert noalloc(H=None) == 1 and noalloc(lp=2050) == 1
    # beyond the fixed 32 MiB scratch: 4 n (2 ceil(V / 2048) + 1) bytes plus the status word
    assert noalloc(n=1 << 20, V=151936) == 3

    def after_timeout(**kw):
        a = dict(use=0, H=256, W=512, ids=1024, n=100, d=256, V=4096, lp=2048, lse=None, ws=1 << 20, wsb=1 << 40)
        a.update(kw)
        return lib.rz_selftest_forward_after_timeout(a["use"], a["H"], a["W"], a["ids"], a["n"], a["d"], a["V"],
                                                     a["lp"], a["lse"], a["ws"], a["wsb"], None)

    # the same host checks as the call each variant runs
    assert after_timeout(n=-1) == 1 and after_timeout(d=96) == 2 and after_timeout(H=None) == 1
    assert after_timeout(ws=None) == 1 and after_timeout(ws=(1 << 20) + 16) == 1 and after_timeout(wsb=100) == 3
    assert after_timeout(use=1, ws=None, wsb=0, n=1 << 20, V=151936) == 3
    assert after_timeout(n=0, H=None, W=None, ids=None, lp=None, ws=None) == 0

    count = ctypes.c_int32(-5)
    kinds = (ctypes.c_int32 * 4)()
    events = (ctypes.c_void_p * 8)()

    def timed(n=100, ev=events, cap=4):
        return lib.rz_loss_fwd_bwd_timed(256, 512, 1024, 2048, 3072, 4096, 5120, n, 4, 2, 256, 4096, 6144, 7168,
                                         8192, None, None, 1 << 20, 1 << 40, None, ev, kinds, cap,
                                         ctypes.byref(count))

    assert timed(ev=None) == 1 and timed(cap=-1) == 1
    assert timed(n=0) == 1 and count.value == 0   # nothing recorded on an argument error
    assert lib.rz_num_launches_loss(0) == 0
    # the loss setup, then 6 per 16384-token chunk
    assert [lib.rz_num_launches_loss(n) for n in (1, 16384, 16385)] == [7, 7, 13]
    assert lib.rz_read_device_status(None, None, None) == 1
