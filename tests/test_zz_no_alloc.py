"""awq_search_noalloc: the search for callers that cannot allocate device
memory (an engine or plugin host that owns all device memory, a real-time path
with a fixed memory budget).  Its scratch space is a fixed-size device array
inside the library, so the call needs no workspace argument.

The test calls the entry point through the C ABI and checks it against
awq_search with a caller workspace, within the search's tolerance (relative
1e-2 on every L(alpha), identical alpha*), on two calls in a row: the second
call finds the first call's leftovers in the shared scratch.  This file is
collected last so that a failing run that stops at the first failure has run
every other test already; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

L_RTOL = 1e-2
AWQ_EWORKSPACE = 4
SCRATCH_BYTES = 32 << 20


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from post_weight_only_b200 import awq
    fn = awq._lib.awq_search_noalloc
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fn.argtypes = [P, P, P, I64, I64, I64, P, I, I, I, I, P, P, P, P, P, P]
    fn.restype = I
    return awq, fn


def _noalloc(awq, fn, X, W, a, grid, bits, group, form):
    N, D_in = X.shape
    D_out = W.shape[1]
    A = len(grid)
    g = (ctypes.c_float * A)(*grid)
    L = torch.empty(A, dtype=torch.float64, device="cuda")
    Lc = torch.empty(A, D_out, dtype=torch.float64, device="cuda")
    astar = torch.empty(1, dtype=torch.float32, device="cuda")
    aidx = torch.empty(1, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    rc = fn(X.data_ptr(), W.data_ptr(), a.data_ptr(), N, D_in, D_out, g, A, bits, group, form, L.data_ptr(),
            Lc.data_ptr(), astar.data_ptr(), aidx.data_ptr(), status.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    assert rc == 0, awq.last_error()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return L.cpu().numpy(), Lc.cpu().numpy(), float(astar.item()), int(aidx.item())


@pytest.mark.parametrize("form", ["error", "reference"])
@pytest.mark.parametrize("N,D_in,D_out,bits,group", [(256, 512, 512, 4, 128), (300, 384, 200, 3, 64)])
def test_noalloc_matches_workspace_search_twice(lib, form, N, D_in, D_out, bits, group):
    awq, fn = lib
    fid = awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE
    X, W = synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=7))
    Xd, Wd = X.cuda(), W.cuda()
    a = awq.act_stats(Xd)
    grid = synth.alpha_grid(20).tolist()
    ref = awq.search(Xd, Wd, a, grid, bits, group, want_cols=True, loss_form=fid)
    L_ref, Lc_ref = ref.L.cpu().numpy(), ref.L_col.cpu().numpy()
    for _ in range(2):
        L, Lc, astar, aidx = _noalloc(awq, fn, Xd, Wd, a, grid, bits, group, fid)
        assert np.allclose(L, L_ref, rtol=L_RTOL, atol=0)
        assert np.allclose(Lc, Lc_ref, rtol=L_RTOL, atol=1e-30)
        assert aidx == int(ref.alpha_idx.item())
        assert astar == float(ref.alpha_star.item())


def test_noalloc_rejects_shapes_beyond_the_scratch(lib):
    awq, fn = lib
    # 4096 x 4096 with 21 alphas needs far more than the built-in scratch.
    N, D_in, D_out = 4096, 4096, 4096
    need = awq.search_workspace_size(N, D_in, D_out, 21, 4, 128)
    assert need > SCRATCH_BYTES
    X = torch.zeros(16, D_in, dtype=torch.bfloat16, device="cuda")     # never read: rejected first
    W = torch.zeros(16, D_out, dtype=torch.float32, device="cuda")
    a = torch.ones(D_in, dtype=torch.float32, device="cuda")
    g = (ctypes.c_float * 21)(*synth.alpha_grid(20).tolist())
    out = torch.empty(64, dtype=torch.float64, device="cuda")
    rc = fn(X.data_ptr(), W.data_ptr(), a.data_ptr(), N, D_in, D_out, g, 21, 4, 128, 0, out.data_ptr(), None,
            out.data_ptr(), out.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert rc == AWQ_EWORKSPACE
    msg = awq.last_error()
    assert str(need) in msg and str(SCRATCH_BYTES) in msg
