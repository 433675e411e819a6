"""The C ABI: the library builds, loads on a machine without a GPU, and exports
every entry point that include/mk.h declares."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "mk.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mk_create", "mk_build_schedule", "mk_decode_step", "mk_baseline_decode_step",
                     "mk_decode_step_host", "mk_get_status", "mk_destroy", "mk_status_str"):
        assert required in names


def test_library_exports_every_declared_symbol():
    from persistent_megakernel_interpreter_b200 import _lib
    lib = _lib.lib()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_struct_sizes():
    from persistent_megakernel_interpreter_b200 import _lib
    lib = _lib.lib()
    assert lib.mk_status_str(0) == b"ok"
    assert lib.mk_status_str(5) == b"device wait timed out"
    assert ctypes.sizeof(_lib.MkInstr) == 48
    # null handles are rejected, not dereferenced
    assert lib.mk_decode_step(None, None, None, None, None, None, None) == 1
    assert lib.mk_build_schedule(None, 1, 1, None) == 1
    lib.mk_destroy(None)
    # greedy selection: null buffers and empty sizes are refused before any launch
    fake = ctypes.c_void_p(256)
    assert lib.mk_greedy_select(None, 1, 8, fake, None, None) == 1
    assert lib.mk_greedy_select(fake, 1, 8, None, None, None) == 1
    assert lib.mk_greedy_select(fake, 0, 8, fake, None, None) == 1
    assert lib.mk_greedy_select(fake, 1, 0, fake, None, None) == 1


def test_create_rejects_unsupported_shapes():
    from persistent_megakernel_interpreter_b200 import _lib
    from persistent_megakernel_interpreter_b200.config import TINY
    import dataclasses
    lib = _lib.lib()
    bad = dataclasses.replace(TINY, head_dim=96)
    c = _lib.make_config(bad, 1, 16)
    assert lib.mk_packed_bytes(ctypes.byref(c)) == 0
    w = _lib.MkWeights()
    h = ctypes.c_void_p()
    assert lib.mk_create(ctypes.byref(c), ctypes.byref(w), 0, ctypes.byref(h)) == 3
    assert not h.value
    # dimensions far above any model are refused before any size is computed from them
    for field, value in (("hidden", 1 << 29), ("ffn", 1 << 30), ("vocab", 1 << 30)):
        c = _lib.make_config(dataclasses.replace(TINY, **{field: value}), 1, 16)
        assert lib.mk_packed_bytes(ctypes.byref(c)) == 0, field
    assert lib.mk_packed_bytes(ctypes.byref(_lib.make_config(TINY, 1, (1 << 20) + 1))) == 0
    assert lib.mk_packed_bytes(ctypes.byref(_lib.make_config(TINY, 1, 1 << 20))) > 0


def test_header_is_plain_c_and_a_c_program_links_against_the_library(tmp_path):
    """include/mk.h compiles as C99 with warnings as errors, and a C program that
    takes the address of every declared entry point links against libmk.so."""
    import shutil
    import subprocess
    from persistent_megakernel_interpreter_b200 import build
    gcc = shutil.which("gcc")
    if gcc is None:
        import pytest
        pytest.skip("gcc not available")
    names = declared_functions()
    src = tmp_path / "use_mk.c"
    src.write_text("#include \"mk.h\"\n#include <stdio.h>\n"
                   "typedef void (*any_fn)(void);\n"
                   "int main(void) {\n"
                   "    any_fn fns[] = {" + ", ".join(f"(any_fn)&{n}" for n in names) + "};\n"
                   "    printf(\"%d %s\\n\", (int)(sizeof fns / sizeof fns[0]), mk_status_str(MK_OK));\n"
                   "    return 0;\n}\n")
    exe = tmp_path / "use_mk"
    libdir = os.path.dirname(build.LIB)
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           f"-I{os.path.join(ROOT, 'include')}", str(src), "-o", str(exe),
                           f"-L{libdir}", "-l:libmk.so", f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out == [str(len(names)), "ok"]


def test_ctypes_declarations_match_the_c_header(tmp_path):
    """Every ctypes structure of the binding has the size and field offsets the C
    compiler gives the header's struct, and the status and opcode numbers agree."""
    import shutil
    import subprocess
    from persistent_megakernel_interpreter_b200 import _lib
    gcc = shutil.which("gcc")
    if gcc is None:
        import pytest
        pytest.skip("gcc not available")
    structs = {"mk_config": _lib.MkConfig, "mk_weights": _lib.MkWeights,
               "mk_schedule_opts": _lib.MkScheduleOpts, "mk_instr": _lib.MkInstr,
               "mk_schedule_info": _lib.MkScheduleInfo}
    lines = []
    want = []
    for cname, py in structs.items():
        lines.append(f'printf("%zu\\n", sizeof({cname}));')
        want.append(ctypes.sizeof(py))
        for fname, _ in py._fields_:
            lines.append(f'printf("%zu\\n", offsetof({cname}, {fname}));')
            want.append(getattr(py, fname).offset)
    for code, name in sorted(_lib.STATUS.items()):
        lines.append(f'printf("%d\\n", (int){name});')
        want.append(code)
    for name in ("QKV", "ATTN", "OPROJ", "GATEUP", "DOWN", "LMHEAD"):
        lines.append(f'printf("%d\\n", (int)MK_OP_{name});')
        want.append(getattr(_lib, f"OP_{name}"))
    lines.append('printf("%u\\n", (unsigned)MK_NO_COUNTER);')
    want.append(_lib.NO_COUNTER)
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"mk.h\"\nint main(void) {\n    "
                   + "\n    ".join(lines) + "\n    return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
                           str(src), "-o", str(exe)])
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert got == want


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: with libmk.so absent, loading raises instead of returning a
    stand-in (the binding's only compute path is the CUDA library)."""
    from persistent_megakernel_interpreter_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libmk.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()
