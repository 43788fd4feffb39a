"""The C-ABI library builds, loads and exports every symbol include/moedec.h
declares; host-side argument checks reject bad calls before any launch. No
compute call is made here (no GPU needed)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    from mixture_experts_decode_moe_b200 import build
    build.build()
    from mixture_experts_decode_moe_b200 import moedec
    return moedec


def declared_functions():
    with open(os.path.join(ROOT, "include", "moedec.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(M):
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(M.EXPORTS)


def test_abi_version_and_status_strings(M):
    assert M.moe_abi_version() == 2
    for s in range(5):
        assert M.moe_status_string(s)
    assert M.moe_status_string(99) == "unknown status"


def desc(M, **kw):
    d = dict(H=2048, E=256, I=512, k=8)
    d.update(kw)
    return M.LayerDesc(d["H"], d["E"], d["I"], d["k"], kw.get("kind", 0), kw.get("wtype", 0),
                       kw.get("layout", 0), kw.get("I_shared", 0))


def test_workspace_bytes_host_side(M):
    a3b = desc(M)
    n1 = M.moe_workspace_bytes(a3b, 1)
    # control block + logits [B, E] fp32 + two fp32 accumulators [B, H]
    assert n1 >= 256 + 1 * 256 * 4 + 2 * 1 * 2048 * 4
    assert M.moe_workspace_bytes(a3b, 8) > n1
    for bad in (desc(M, k=0), desc(M, k=33), desc(M, E=2000), desc(M, H=100), desc(M, k=9, E=8),
                desc(M, wtype=1, H=256), desc(M, wtype=1, I=100), desc(M, kind=7)):
        assert M.moe_workspace_bytes(bad, 1) == 0
    assert M.moe_workspace_bytes(a3b, 0) == 0
    assert M.moe_workspace_bytes(a3b, 257) == 0


def test_invalid_arguments_rejected_before_launch(M):
    lib = M._lib
    P = ctypes.c_void_p
    dummy = P(4096)  # never dereferenced: every call below fails validation first
    assert lib.moe_route_topk(None, dummy, 1, 2048, 256, 8, dummy, dummy, None, dummy, 1 << 20, None) == 1
    assert lib.moe_route_topk(dummy, dummy, 0, 2048, 256, 8, dummy, dummy, None, dummy, 1 << 20, None) == 1
    assert lib.moe_route_topk(dummy, dummy, 1, 2048, 256, 40, dummy, dummy, None, dummy, 1 << 20, None) == 1
    assert lib.moe_route_topk(P(4097), dummy, 1, 2048, 256, 8, dummy, dummy, None, dummy, 1 << 20, None) == 1
    assert lib.moe_touched_experts(None, 1, 2, 16, dummy, None, None, None, None) == 1
    assert lib.moe_touched_experts(dummy, 300, 2, 16, dummy, None, None, None, None) == 1
    d = desc(M)
    assert lib.moe_layer_forward(ctypes.byref(d), dummy, 1, dummy, None, None, None, dummy, 1 << 20,
                                 None) == 1  # no weights
    assert lib.moe_stack_forward(ctypes.byref(d), 0, dummy, 1, 0, dummy, None, None, None, None, dummy,
                                 1 << 20, None) == 1
    assert lib.moe_stack_forward(ctypes.byref(d), 1, dummy, 1, 2, dummy, None, None, None, None, dummy,
                                 1 << 20, None) == 1  # unknown flag
    assert lib.moe_workspace_init(None, 0, None) == 1
    assert lib.moe_get_status(None, None) == 1
    cm = desc(M, E=128, I=768, layout=1)
    assert lib.moe_channel_topk_forward(ctypes.byref(cm), dummy, 1, dummy, dummy, dummy, 8 * 768 + 1,
                                        dummy, None, dummy, None, None, dummy, 1 << 20, None) == 1
    # batches of more than 8 tokens are rejected
    assert lib.moe_channel_topk_forward(ctypes.byref(cm), dummy, 9, dummy, dummy, dummy, 10,
                                        dummy, None, dummy, None, None, dummy, 1 << 30, None) == 1


def test_reader_entries_reject_bad_arguments_before_launch(M):
    lib = M._lib
    P = ctypes.c_void_p
    dummy = P(4096)  # never dereferenced: every call below fails validation first
    cm = desc(M, E=128, I=768, layout=1)
    cm.gate = dummy
    planar = desc(M, E=128, I=768)
    planar.gate = dummy
    odd_h = desc(M, H=192, E=16, I=64, k=2, layout=1)  # H % 128 != 0
    odd_h.gate = dummy
    wide = desc(M, H=4096, E=16, I=64, k=2, layout=1)
    wide.gate = dummy
    b = ctypes.byref
    assert lib.moe_reader_build(b(planar), dummy, dummy, dummy, dummy, dummy, None) == M.MOE_ERR_INVALID
    assert lib.moe_reader_build(b(cm), None, dummy, dummy, dummy, dummy, None) == M.MOE_ERR_INVALID
    assert lib.moe_reader_build(b(cm), dummy, P(4098), dummy, dummy, dummy, None) == M.MOE_ERR_INVALID
    assert lib.moe_reader_build(b(odd_h), dummy, dummy, dummy, dummy, dummy, None) == M.MOE_ERR_UNSUPPORTED
    assert lib.moe_reader_build(b(wide), dummy, dummy, dummy, dummy, dummy, None) == M.MOE_ERR_UNSUPPORTED
    args = (dummy, dummy, dummy, dummy, dummy, dummy, dummy, None, None)
    assert lib.moe_reader_screen(b(cm), dummy, 0, *args) == M.MOE_ERR_INVALID
    assert lib.moe_reader_screen(b(cm), dummy, 257, *args) == M.MOE_ERR_INVALID
    assert lib.moe_reader_screen(b(planar), dummy, 1, *args) == M.MOE_ERR_INVALID
    assert lib.moe_reader_screen(b(cm), None, 1, *args) == M.MOE_ERR_INVALID
    assert lib.moe_reader_screen(b(odd_h), dummy, 1, *args) == M.MOE_ERR_UNSUPPORTED


def test_plain_c_program_links_and_calls_the_abi(M, tmp_path):
    """The boundary is usable from C: the header compiles as C99, and a C
    program linked against libmoedec.so gets the ABI version and a host-side
    argument rejection (no GPU work)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        '#include <stdio.h>\n#include "moedec.h"\n'
        "int main(void) {\n"
        "  moe_layer_desc d = {0};\n"
        "  moe_status st = moe_layer_forward(&d, 0, 1, 0, 0, 0, 0, 0, 0, 0);\n"
        '  printf("%d %d %s\\n", moe_abi_version(), (int)st, moe_status_string(st));\n'
        "  return 0;\n}\n")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(M.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-l:" + os.path.basename(M.LIB_PATH), "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out[0] == "2" and out[1] == str(M.MOE_ERR_INVALID)


def test_budget_and_injection_reject_bad_arguments_before_launch(M):
    lib = M._lib
    P = ctypes.c_void_p
    assert lib.moe_workspace_set_wait_budget(None, 5, None) == M.MOE_ERR_INVALID
    assert lib.moe_workspace_set_wait_budget(P(4097), 5, None) == M.MOE_ERR_INVALID
    assert lib.moe_workspace_set_inject(None, 1, None) == M.MOE_ERR_INVALID
    assert lib.moe_workspace_set_inject(P(4096), 2, None) == M.MOE_ERR_INVALID  # unknown bit
