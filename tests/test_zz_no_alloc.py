"""w4a8_gemm_static_scratch, the entry point that allocates nothing: it must
give what w4a8_gemm gives (the same kernels, its split-K partials in the
library's fixed per-device buffer instead of a caller workspace), call after
call, and reject shapes whose scratch exceeds the fixed size.

Collected last on purpose (file name), so it also runs after every other GPU
test has used the library in the same process."""
import ctypes

import numpy as np
import pytest
import torch

from synth import gen_linear
from tests._util import bits

pytestmark = pytest.mark.gpu

W4A8_ERR_WORKSPACE = 7
STATIC_SCRATCH_BYTES = 8 << 20  # W4A8_STATIC_SCRATCH_BYTES in include/w4a8.h


@pytest.fixture(scope="module")
def m():
    from moe_linear_layers_w4a8_b200 import _build
    _build.build()
    import moe_linear_layers_w4a8_b200 as mm
    mm.load_library()
    return mm


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _static_call(m, qx, s_x, w, Y, status):
    """One call of the C ABI entry point; returns its status code."""
    L = m.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream(qx.device).cuda_stream)
    return int(L.w4a8_gemm_static_scratch(_p(qx), _p(s_x), _p(w.packed), _p(w.s_w), _p(w.z),
                                          ctypes.byref(w.desc), qx.shape[0], _p(Y), Y.stride(0),
                                          _p(status), stream))


def _same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    return bool(np.array_equal(bits(a), bits(b)))


@pytest.mark.parametrize("M,K,N,group,sym", [
    (32, 4096, 14336, 128, True),   # decode shape, split-K, ~5.5 MB of scratch
    (8, 4096, 14336, 128, True),
    (16, 512, 512, 128, True),      # small, several groups per tile split across CTAs
    (5, 2048, 1024, 64, False),     # asymmetric, group 64, ragged M
])
def test_static_scratch_matches_workspace_entry(m, M, K, N, group, sym):
    torch.manual_seed(0)
    a = gen_linear(M, K, N, seed=11)
    b = gen_linear(M, K, N, seed=12)
    w = m.w4a8_pack_weights(a.W.cuda(), group, sym)
    need = m.w4a8_gemm_workspace_size(M, w)
    assert 0 < need <= STATIC_SCRATCH_BYTES
    qa, sa, _ = m.w4a8_quant_act(a.X.cuda())
    qb, sb, _ = m.w4a8_quant_act(b.X.cuda())
    ref_a = m.w4a8_gemm(qa, sa, w)
    ref_b = m.w4a8_gemm(qb, sb, w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two calls in a row, different activations, the same scratch buffer
    Ya = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    Yb = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _static_call(m, qa, sa, w, Ya, status) == 0
    assert _static_call(m, qb, sb, w, Yb, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # the same kernels, plan and fixed split-K summation order as the workspace
    # entry point: bit for bit its results
    assert _same_bits(Ya, ref_a)
    assert _same_bits(Yb, ref_b)
    # and again on the first input, after the buffer held the second call's partials
    Ya2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _static_call(m, qa, sa, w, Ya2, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert _same_bits(Ya2, ref_a)


def test_static_scratch_rejects_oversize(m):
    M, K, N = 64, 4096, 14336
    a = gen_linear(M, K, N, seed=13)
    w = m.w4a8_pack_weights(a.W.cuda(), 128, True)
    need = m.w4a8_gemm_workspace_size(M, w)
    if need <= STATIC_SCRATCH_BYTES:
        pytest.skip(f"this GPU's plan needs only {need} bytes at M={M}")
    qx, s_x, _ = m.w4a8_quant_act(a.X.cuda())
    Y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _static_call(m, qx, s_x, w, Y, status) == W4A8_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert int(torch.count_nonzero(Y).item()) == 0  # nothing was launched
    with pytest.raises(m.W4A8Error):
        m.w4a8_gemm_static_scratch(qx, s_x, w, out=Y)
