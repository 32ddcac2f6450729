"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_39_b200 import _lib
from block_sparse_attention_39_b200 import pbsa as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "pbsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pbsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = header_functions()
    for n in ["pbsa_score_blocks", "pbsa_update_memory", "pbsa_select_local", "pbsa_attn_fwd",
              "pbsa_attn_bwd", "pbsa_get_status"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    missing = [n for n in header_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(header_functions()) == set(_lib.SIGNATURES)


def test_version_and_last_error():
    assert "sm_100a" in K.version()
    assert isinstance(_lib.lib().pbsa_last_error(), bytes)


def _d(**kw):
    base = dict(B=1, H=2, D=128, bs=128, scale=0.088, dtype=0)
    base.update(kw)
    return _lib.PbsaDims(**base)


NULL = None


@pytest.mark.parametrize("kw,code", [(dict(D=96), -2), (dict(bs=32), -2), (dict(B=0), -2),
                                     (dict(dtype=7), -4)])
def test_bad_dims_rejected_without_launch(kw, code):
    lib = _lib.lib()
    d = _d(**kw)
    rc = lib.pbsa_score_blocks(ctypes.byref(d), NULL, 10, NULL, 4, NULL, NULL, 0, NULL, NULL, NULL,
                               NULL, NULL)
    assert rc == code
    assert lib.pbsa_last_error()


def test_null_buffers_rejected():
    lib = _lib.lib()
    d = _d()
    assert lib.pbsa_score_blocks(ctypes.byref(d), NULL, 10, NULL, 4, NULL, NULL, 0, NULL, NULL,
                                 NULL, NULL, NULL) == -1
    assert lib.pbsa_attn_fwd(ctypes.byref(d), NULL, 10, 0, NULL, NULL, 4, NULL, NULL, NULL, NULL,
                             4, 0, NULL, NULL, NULL) == -1
    assert lib.pbsa_select_local(ctypes.byref(d), NULL, 1, 4, NULL, 0, 1, NULL, 0, 0, NULL, 0, 0,
                                 NULL, 10, NULL, NULL, 4, 0, 1, NULL) == -1


def test_attention_rejects_fp32():
    lib = _lib.lib()
    d = _d(dtype=1)
    assert lib.pbsa_attn_fwd(ctypes.byref(d), NULL, 10, 0, NULL, NULL, 4, NULL, NULL, NULL, NULL,
                             4, 0, NULL, NULL, NULL) == -4


def test_update_limits_and_workspace_size():
    lib = _lib.lib()
    d = _d()
    fake = ctypes.c_void_p(256)       # never dereferenced: validation fails first
    # P > 256
    assert lib.pbsa_update_memory(ctypes.byref(d), fake, fake, 400, fake, fake, fake, 300, 0,
                                  fake, fake, fake, fake, 1, fake, 0, fake, 1 << 30, NULL) == -2
    # too many candidates
    assert lib.pbsa_update_memory(ctypes.byref(d), fake, fake, 400, fake, fake, fake, 64, 0,
                                  fake, fake, fake, fake, 200, fake, 0, fake, 1 << 30, NULL) == -2
    need = K.update_memory_workspace(d, 24, 111)
    assert need > 0 and need % 256 == 0
    # workspace too small
    assert lib.pbsa_update_memory(ctypes.byref(d), fake, fake, 209, fake, fake, fake, 24, 0,
                                  fake, fake, fake, fake, 111, fake, 0, fake, need - 1, NULL) == -7
    # bad policy
    assert lib.pbsa_update_memory(ctypes.byref(d), fake, fake, 209, fake, fake, fake, 24, 0,
                                  fake, fake, fake, fake, 111, fake, 5, fake, need, NULL) == -1


def test_select_limits():
    lib = _lib.lib()
    d = _d()
    fake = ctypes.c_void_p(256)
    # n_mem + min(k, n_win) > Amax
    assert lib.pbsa_select_local(ctypes.byref(d), fake, 1, 300, fake, 74, 16, fake, 24, 0, fake, 0,
                                 0, NULL, 100, fake, fake, 39, 0, 1, NULL) == -2
    # window too long for one warp
    assert lib.pbsa_select_local(ctypes.byref(d), fake, 1, 600, fake, 600, 16, NULL, 0, 0, fake, 0,
                                 0, NULL, 100, fake, fake, 64, 0, 1, NULL) == -2


def test_route_args_layout_matches_the_header(tmp_path):
    # the ctypes mirror of pbsa_route_args must have the C layout: compile a
    # probe against the header with the host compiler and compare offsets
    fields = [n for n, _ in _lib.ROUTE_FIELDS]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "pbsa.h"\nint main(void){\n'
                   + "".join(f'  printf("%zu\\n", offsetof(pbsa_route_args, {n}));\n' for n in fields)
                   + '  printf("%zu\\n", sizeof(pbsa_route_args));\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    want = [getattr(_lib.PbsaRouteArgs, n).offset for n in fields] + [ctypes.sizeof(_lib.PbsaRouteArgs)]
    assert got == want


def test_route_rejects_bad_arguments_without_launch():
    lib = _lib.lib()
    d = _d()
    assert lib.pbsa_route_step(ctypes.byref(d), None, None, 0, None) == -1
    a = _lib.PbsaRouteArgs(Tq=128, NB=8, n_pool=0, P=0, n_cand=0)
    # no workspace
    assert lib.pbsa_route_step(ctypes.byref(d), ctypes.byref(a), None, 0, None) == -7
    # workspace too small: the barrier words alone need 256 bytes
    assert lib.pbsa_route_step(ctypes.byref(d), ctypes.byref(a), ctypes.c_void_p(4096), 128,
                               None) == -7
    a.Tq = 0
    assert lib.pbsa_route_step(ctypes.byref(d), ctypes.byref(a), ctypes.c_void_p(4096), 4096,
                               None) == -2
    assert lib.pbsa_route_workspace(ctypes.byref(d), 0, 0) == 256
    assert (lib.pbsa_route_workspace(ctypes.byref(d), 24, 111)
            == 256 + lib.pbsa_update_memory_workspace(ctypes.byref(d), 24, 111))


def test_append_rejects_bad_arguments_without_launch():
    lib = _lib.lib()
    d = _d()
    fake = ctypes.c_void_p(256)       # never dereferenced: validation fails first
    # NULL buffers
    assert lib.pbsa_append_chunk(ctypes.byref(d), NULL, NULL, 300, 0, NULL, NULL, 8, NULL, NULL,
                                 NULL, NULL, NULL) == -1
    # the chunk (3 blocks of 128) does not fit a 2-block pool
    assert lib.pbsa_append_chunk(ctypes.byref(d), fake, fake, 300, 0, fake, fake, 2, fake, fake,
                                 fake, fake, NULL) == -2
    # empty chunk
    assert lib.pbsa_append_chunk(ctypes.byref(d), fake, fake, 0, 0, fake, fake, 8, fake, fake,
                                 fake, fake, NULL) == -2
    # misaligned K rows
    assert lib.pbsa_append_chunk(ctypes.byref(d), ctypes.c_void_p(264), fake, 300, 0, fake, fake,
                                 8, fake, fake, fake, fake, NULL) == -3


def test_update_bwd_rejects_bad_arguments_without_launch():
    lib = _lib.lib()
    d = _d()
    fake = ctypes.c_void_p(4096)
    assert lib.pbsa_update_memory_bwd(ctypes.byref(d), 64, 24, 37, NULL, fake, fake, fake, 1 << 30,
                                      NULL) == -1
    assert lib.pbsa_update_memory_bwd(ctypes.byref(d), 8, 24, 37, fake, fake, fake, fake, 1 << 30,
                                      NULL) == -2            # NB < P
    assert lib.pbsa_update_memory_bwd(ctypes.byref(d), 64, 24, 37, fake, ctypes.c_void_p(4100),
                                      fake, fake, 1 << 30, NULL) == -3
    need = lib.pbsa_update_memory_bwd_workspace(ctypes.byref(d), 24)
    assert need == 2 * 24 * 2 * 128 * 128 * 4
    assert lib.pbsa_update_memory_bwd(ctypes.byref(d), 64, 24, 37, fake, fake, fake, fake,
                                      need - 1, NULL) == -7
    # the plan is the head of the update workspace
    assert 0 < lib.pbsa_update_plan_bytes(ctypes.byref(d), 24, 37) <= \
        lib.pbsa_update_memory_workspace(ctypes.byref(d), 24, 37)
