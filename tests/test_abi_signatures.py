"""The Python binding's ctypes signatures agree with include/rz.h, parameter by parameter
(CPU only, nothing is called): a 32-bit integer where the header has a 64-bit one, or a
missing parameter, would shift every argument after it without any error.  Also the
rz_loss_options layout (against offsetof/sizeof from the C compiler on this header), the
status codes and the option flags."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rz.h")

SCALARS = {"int64_t": ctypes.c_int64, "int32_t": ctypes.c_int32, "size_t": ctypes.c_size_t,
           "uint64_t": ctypes.c_uint64, "int": ctypes.c_int, "rz_status": ctypes.c_int, "float": ctypes.c_float,
           "double": ctypes.c_double}


def _header_text():
    return re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)


def _prototypes():
    """name -> (return type, [parameter types]) of every rz_* function the header declares."""
    out = {}
    for m in re.finditer(r"([A-Za-z_][A-Za-z0-9_ ]*\**)\s+\**\s*(rz_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", _header_text()):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3)
        ps = [] if params.strip() in ("", "void") else [p.strip() for p in params.split(",")]
        types = []
        for p in ps:
            p = re.sub(r"\s+", " ", p)
            if "*" in p:
                types.append("ptr")
            else:
                base = p.replace("const ", "").rsplit(" ", 1)[0]
                types.append(SCALARS[base])
        out[name] = (ret, types)
    return out


def _is_pointer(t):
    return t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer))


@pytest.fixture(scope="module")
def lib():
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    import invariant_logprobs_reinforce_b200 as rz
    return rz.lib()


def test_every_prototype_is_parsed():
    protos = _prototypes()
    import invariant_logprobs_reinforce_b200 as rz
    assert set(protos) == set(rz.EXPORTED_SYMBOLS)


def test_every_declared_call_has_a_python_function_of_the_same_name():
    import invariant_logprobs_reinforce_b200 as rz
    missing = [name for name in _prototypes() if not callable(getattr(rz, name, None))]
    assert not missing, missing
    assert set(_prototypes()) <= set(rz.__all__)


@pytest.mark.parametrize("name", sorted(_prototypes()))
def test_binding_signature_matches_the_header(lib, name):
    ret, params = _prototypes()[name]
    fn = getattr(lib, name)
    assert fn.argtypes is not None, f"{name} has no argtypes in the binding"
    assert len(fn.argtypes) == len(params), (name, len(fn.argtypes), len(params))
    for i, (have, want) in enumerate(zip(fn.argtypes, params)):
        if want == "ptr":
            assert _is_pointer(have), (name, i, have)
        else:
            assert have is want, (name, i, have, want)
    want_ret = {"rz_status": ctypes.c_int, "size_t": ctypes.c_size_t, "int32_t": ctypes.c_int32,
                "const char*": ctypes.c_char_p}[ret]
    assert fn.restype is want_ret, (name, fn.restype, want_ret)


def test_loss_options_layout_matches_the_c_compiler(tmp_path):
    import invariant_logprobs_reinforce_b200 as rz
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "rz.h"\n'
        "int main(void) {\n"
        '  printf("%zu %zu %zu %zu %zu %zu %zu\\n", sizeof(rz_loss_options),\n'
        "         offsetof(rz_loss_options, flags), offsetof(rz_loss_options, clip_max),\n"
        "         offsetof(rz_loss_options, gate_lo), offsetof(rz_loss_options, gate_hi),\n"
        "         offsetof(rz_loss_options, token_mask), offsetof(rz_loss_options, n_resp_total));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    size, *offs = map(int, subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split())
    O = rz.rz_loss_options
    assert ctypes.sizeof(O) == size
    assert [getattr(O, f).offset for f in ("flags", "clip_max", "gate_lo", "gate_hi", "token_mask",
                                           "n_resp_total")] == offs


def test_status_codes_and_flags_match_the_header():
    import invariant_logprobs_reinforce_b200 as rz
    text = _header_text()
    enum = dict((k, int(v)) for k, v in re.findall(r"\b(RZ_[A-Z_]+)\s*=\s*(\d+)", text))
    assert {v: k for k, v in enum.items()} == rz.STATUS_NAMES
    flags = dict((k, int(v)) for k, v in re.findall(r"#define\s+(RZ_LOSS_[A-Z_]+)\s+(\d+)", text))
    assert flags == {"RZ_LOSS_CLIP_IS": rz.RZ_LOSS_CLIP_IS, "RZ_LOSS_SEQ_GATE": rz.RZ_LOSS_SEQ_GATE,
                     "RZ_LOSS_TOKEN_MASK": rz.RZ_LOSS_TOKEN_MASK}
