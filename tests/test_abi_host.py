"""C-ABI checks that need no GPU: the library builds and loads, exports every
function include/w4a8.h declares, and rejects bad arguments on the host
(before any CUDA call) with the documented status codes."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from moe_linear_layers_w4a8_b200 import _build
    _build.build()
    import moe_linear_layers_w4a8_b200 as m
    return m.load_library()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "w4a8.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:w4a8|w8a8|w4a16)_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared_functions()
    for required in ("w4a8_pack_weights", "w4a8_quant_act", "w4a8_gemm", "w4a8_moe_grouped_gemm",
                     "w8a8_gemm", "w4a16_gemm"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_exports_nothing_else(lib):
    import subprocess
    from moe_linear_layers_w4a8_b200 import library_path
    out = subprocess.run(["nm", "-D", "--defined-only", library_path()], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {n for n in exported if n.startswith(("w4a8_", "w8a8_", "w4a16_"))}
    assert ours == set(_declared_functions())


def test_status_strings(lib):
    import moe_linear_layers_w4a8_b200 as m
    assert lib.w4a8_abi_version() == 1
    for code, name in m.STATUS.items():
        assert m.w4a8_status_string(code) == name


def _desc(**kw):
    import moe_linear_layers_w4a8_b200 as m
    d = dict(bits=4, symmetric=1, group=128, K=512, N=512, layout_version=1)
    d.update(kw)
    return m.WDesc(**d)


def test_sizes(lib):
    import moe_linear_layers_w4a8_b200 as m
    assert lib.w4a8_packed_bytes(4096, 14336) == 4096 * 14336 // 2
    assert lib.w4a8_packed_bytes(0, 5) == 0
    d = _desc()
    assert lib.w4a8_gemm_workspace_size(0, ctypes.byref(d)) == 0
    bad = _desc(layout_version=2)
    assert lib.w4a8_gemm_workspace_size(16, ctypes.byref(bad)) == 0
    w1 = _desc(K=2048, N=2816)
    w2 = _desc(K=1408, N=2048)
    lay = m.MoeWsLayout()
    assert lib.w4a8_moe_workspace_layout(4096, 64, 6, ctypes.byref(w1), ctypes.byref(w2), ctypes.byref(lay)) == 0
    assert lay.total == lib.w4a8_moe_workspace_size(4096, 64, 6, ctypes.byref(w1), ctypes.byref(w2))
    offs = [lay.perm, lay.inv, lay.qx, lay.sx, lay.h, lay.qh, lay.sh, lay.yd]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    R = 4096 * 6
    assert lay.total >= lay.yd + 2 * R * 2048


FAKE = ctypes.c_void_p(256)  # never dereferenced: every case below fails its host check first


@pytest.mark.parametrize("kw,code", [
    (dict(layout_version=2), 3), (dict(bits=8), 3), (dict(group=32), 3), (dict(N=100), 3),
    (dict(K=500), 3), (dict(symmetric=2), 3),
])
def test_gemm_rejects_bad_descriptor(lib, kw, code):
    d = _desc(**kw)
    r = lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(d), 16, FAKE, 512, None, 0, None, None)
    assert r == code


def test_gemm_rejects_zero_point_mismatch(lib):
    d = _desc(symmetric=1)
    assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(d), 16, FAKE, 512, None, 0, None, None) == 3
    d = _desc(symmetric=0)
    assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(d), 16, FAKE, 512, None, 0, None, None) == 3


def test_gemm_rejects_bad_args(lib):
    d = _desc()
    assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(d), -1, FAKE, 512, None, 0, None, None) == 1
    assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(d), 16, FAKE, 100, None, 0, None, None) == 1
    assert lib.w4a8_gemm(None, FAKE, FAKE, FAKE, None, ctypes.byref(d), 16, FAKE, 512, None, 0, None, None) == 1
    assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, None, 16, FAKE, 512, None, 0, None, None) == 1
    # M == 0 is a no-op
    assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(d), 0, FAKE, 512, None, 0, None, None) == 0
    assert lib.w4a8_gemm_debug_partials(FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(d), 16, FAKE, 512, None,
                                        None, 0, None, None) == 1


def test_linear_sizes_and_rejections(lib):
    d = _desc()
    need = lib.w4a8_linear_workspace_size(16, ctypes.byref(d))
    assert need >= 16 * 512 + 16 * 4                       # q_x and s_x at least
    assert lib.w4a8_linear_workspace_size(0, ctypes.byref(d)) == 0
    bad = _desc(layout_version=2)
    assert lib.w4a8_linear(FAKE, 16, 512, FAKE, FAKE, None, ctypes.byref(bad), FAKE, 512, FAKE, need, None, None) == 3
    assert lib.w4a8_linear(FAKE, 16, 512, FAKE, FAKE, None, ctypes.byref(d), FAKE, 512, FAKE, need - 1, None, None) == 7
    assert lib.w4a8_linear(FAKE, 16, 100, FAKE, FAKE, None, ctypes.byref(d), FAKE, 512, FAKE, need, None, None) == 1
    assert lib.w4a8_linear(FAKE, 16, 512, FAKE, FAKE, None, ctypes.byref(d), FAKE, 100, FAKE, need, None, None) == 1
    assert lib.w4a8_linear(FAKE, -1, 512, FAKE, FAKE, None, ctypes.byref(d), FAKE, 512, FAKE, need, None, None) == 1
    assert lib.w4a8_linear(FAKE, 0, 512, FAKE, FAKE, None, ctypes.byref(d), FAKE, 512, FAKE, 0, None, None) == 0


def test_w4a16_sizes_and_rejections(lib):
    d = _desc()
    need = lib.w4a16_gemm_workspace_size(16, ctypes.byref(d))
    # split-K partials only when the tiles leave SMs idle: with no GPU to ask
    # the SM count is taken as 1 and the plan needs no workspace
    assert lib.w4a16_gemm_workspace_size(0, ctypes.byref(d)) == 0
    bad = _desc(layout_version=2)
    assert lib.w4a16_gemm_workspace_size(16, ctypes.byref(bad)) == 0
    args = lambda **k: dict(dict(X=FAKE, M=16, ldx=512, z=None, d=d, ldy=512, ws=FAKE, wsb=need), **k)

    def call(**k):
        a = args(**k)
        return lib.w4a16_gemm(a["X"], a["M"], a["ldx"], FAKE, FAKE, a["z"], ctypes.byref(a["d"]) if a["d"] else None,
                              FAKE, a["ldy"], a["ws"], a["wsb"], None, None)
    assert call(d=bad) == 3
    assert call(z=FAKE) == 3                               # symmetric weight with zero-points
    assert call(d=_desc(symmetric=0)) == 3                 # asymmetric weight without them
    assert call(d=_desc(bits=8)) == 3
    assert call(M=-1) == 1
    assert call(ldy=100) == 1
    assert call(ldx=500) == 1                              # ldx < K
    assert call(ldx=516) == 1                              # row stride not a multiple of 16 bytes
    assert call(X=None) == 1
    assert call(X=ctypes.c_void_p(264)) == 1               # not 16-byte aligned
    if need > 0:
        assert call(wsb=need - 1) == 7
        assert call(ws=None, wsb=0) == 7
    assert call(M=0) == 0
    assert call(d=_desc(K=1 << 25, N=64), ldx=1 << 25) == 2


def test_pack_rejects_bad_args(lib):
    d = _desc()
    # K not a multiple of the group ("groups cannot cross rows")
    assert lib.w4a8_pack_weights(FAKE, 500, 512, 128, 1, FAKE, FAKE, None, ctypes.byref(d), None, None) == 1
    assert lib.w4a8_pack_weights(FAKE, 512, 512, 96, 1, FAKE, FAKE, None, ctypes.byref(d), None, None) == 1
    assert lib.w4a8_pack_weights(FAKE, 512, 100, 128, 1, FAKE, FAKE, None, ctypes.byref(d), None, None) == 1
    assert lib.w4a8_pack_weights(FAKE, 512, 512, 128, 0, FAKE, FAKE, None, ctypes.byref(d), None, None) == 1
    assert lib.w4a8_pack_weights(FAKE, 512, 512, 128, 1, FAKE, FAKE, FAKE, ctypes.byref(d), None, None) == 1
    assert lib.w4a8_pack_weights(None, 512, 512, 128, 1, FAKE, FAKE, None, ctypes.byref(d), None, None) == 1


def test_quant_rejects_bad_args(lib):
    assert lib.w4a8_quant_act(FAKE, 4, 512, 100, 0, FAKE, FAKE, None, None, None) == 1      # ldx < K
    assert lib.w4a8_quant_act(FAKE, 4, 500, 512, 0, FAKE, FAKE, None, None, None) == 2      # K % 8
    assert lib.w4a8_quant_act(FAKE, 4, (1 << 24) + 8, (1 << 24) + 8, 0, FAKE, FAKE, None, None, None) == 2  # K > 2^24
    assert lib.w4a8_quant_act(FAKE, 4, 512, 512, 96, FAKE, FAKE, FAKE, None, None) == 1     # bad group
    assert lib.w4a8_quant_act(FAKE, 4, 512, 512, 128, FAKE, FAKE, None, None, None) == 1    # group w/o rowsum
    assert lib.w4a8_quant_act(FAKE, 0, 512, 512, 0, FAKE, FAKE, None, None, None) == 0      # empty


def test_moe_rejects_bad_shapes(lib):
    w1 = _desc(K=2048, N=2816)
    w2 = _desc(K=1408, N=2048)
    args = lambda T, E, k, a, b: (FAKE, FAKE, T, E, k, FAKE, FAKE, None, ctypes.byref(a), FAKE, FAKE, None,
                                  ctypes.byref(b), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, None, None)
    assert lib.w4a8_moe_grouped_gemm(*args(16, 64, 65, w1, w2)) == 1          # topk > E
    assert lib.w4a8_moe_grouped_gemm(*args(16, 1024, 8, w1, w2)) == 2         # too many experts
    assert lib.w4a8_moe_grouped_gemm(*args(16, 64, 6, w1, _desc(K=1408, N=1024))) == 3  # H mismatch
    assert lib.w4a8_moe_grouped_gemm(*args(16, 64, 6, w1, _desc(K=1408, N=2048, group=64))) == 3
    assert lib.w4a8_moe_grouped_gemm(*args(16, 64, 6, w1, _desc(K=1408, N=2048, symmetric=0))) == 3
    assert lib.w4a8_moe_grouped_gemm(*args(0, 64, 6, w1, w2)) == 0            # empty batch
    a = list(args(16, 64, 6, w1, w2))
    a[17] = None  # no workspace
    assert lib.w4a8_moe_grouped_gemm(*a) == 7


def test_selftest_rejects_bad_limit(lib):
    assert lib.w4a8_selftest_bounded_wait(FAKE, 10, None) == 1
    assert lib.w4a8_selftest_bounded_wait(None, 10000, None) == 1


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "moe_linear_layers_w4a8_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt and "orc_" not in txt, f
