"""awq_search_noalloc: the search for callers that cannot allocate device
memory (an engine or plugin host that owns all device memory, a real-time path
with a fixed memory budget).  Its scratch space is a fixed-size device array
inside the library, so the call needs no workspace argument.

The test calls the entry point through the C ABI and checks it against
awq_search with a caller workspace on two calls in a row (the second call finds
the first call's leftovers in the shared scratch).  Both run the same
deterministic kernels on the same inputs, so L(alpha), the per-column losses
and alpha* must be bit-identical.  It also checks both sides of the scratch
limit: the largest shape of a family that fits runs, the next one is rejected.
This file is collected last so that a failing run that stops at the first
failure has run every other test already; it also passes on its own in a fresh
process.
"""
import ctypes

import numpy as np
import pytest
import torch

from post_weight_only_b200 import synth

pytestmark = pytest.mark.gpu

AWQ_EINVAL = 1
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


def _call(fn, X, W, a, grid, bits, group, form, L, Lc, astar, aidx, status):
    N, D_in = X.shape
    D_out = W.shape[1]
    g = (ctypes.c_float * len(grid))(*grid)
    return fn(X.data_ptr(), W.data_ptr(), a.data_ptr(), N, D_in, D_out, g, len(grid), bits, group, form,
              L.data_ptr(), None if Lc is None else Lc.data_ptr(), astar.data_ptr(), aidx.data_ptr(),
              None if status is None else status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _noalloc(awq, fn, X, W, a, grid, bits, group, form):
    A, D_out = len(grid), W.shape[1]
    L = torch.empty(A, dtype=torch.float64, device="cuda")
    Lc = torch.empty(A, D_out, dtype=torch.float64, device="cuda")
    astar = torch.empty(1, dtype=torch.float32, device="cuda")
    aidx = torch.empty(1, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    rc = _call(fn, X, W, a, grid, bits, group, form, L, Lc, astar, aidx, status)
    assert rc == 0, awq.last_error()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return L.cpu().numpy(), Lc.cpu().numpy(), float(astar.item()), int(aidx.item())


def _check_against_workspace_search(awq, fn, N, D_in, D_out, bits, group, fid, seed=7):
    X, W = synth.layer_inputs(synth.small_layer(N, D_in, D_out, seed=seed))
    Xd, Wd = X.cuda(), W.cuda()
    a = awq.act_stats(Xd)
    grid = synth.alpha_grid(20).tolist()
    ref = awq.search(Xd, Wd, a, grid, bits, group, want_cols=True, loss_form=fid)
    L_ref, Lc_ref = ref.L.cpu().numpy(), ref.L_col.cpu().numpy()
    for _ in range(2):
        L, Lc, astar, aidx = _noalloc(awq, fn, Xd, Wd, a, grid, bits, group, fid)
        assert np.array_equal(L, L_ref)
        assert np.array_equal(Lc, Lc_ref)
        assert aidx == int(ref.alpha_idx.item())
        assert astar == float(ref.alpha_star.item())


@pytest.mark.parametrize("form", ["error", "reference"])
@pytest.mark.parametrize("N,D_in,D_out,bits,group", [(256, 512, 512, 4, 128), (300, 384, 200, 3, 64)])
def test_noalloc_matches_workspace_search_twice(lib, form, N, D_in, D_out, bits, group):
    awq, fn = lib
    fid = awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE
    _check_against_workspace_search(awq, fn, N, D_in, D_out, bits, group, fid)


def _largest_fitting_d_out(awq, N, D_in, A, bits, group, form):
    """The largest D_out (a multiple of 4) whose workspace fits the scratch."""
    lo, hi = 4, 4
    while awq.search_workspace_size(N, D_in, hi, A, bits, group, form) <= SCRATCH_BYTES:
        lo, hi = hi, hi * 2
    while hi - lo > 4:
        mid = (lo + hi) // 2 // 4 * 4
        if awq.search_workspace_size(N, D_in, mid, A, bits, group, form) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return lo


@pytest.mark.parametrize("form", ["error", "reference"])
def test_noalloc_scratch_boundary(lib, form):
    """The largest layer of the family (N = 256, D_in = 512, 21 alphas) that
    fits the scratch runs and matches awq_search; the next size up (D_out + 4)
    is rejected with AWQ_EWORKSPACE before any work."""
    awq, fn = lib
    fid = awq.LOSS_ERROR if form == "error" else awq.LOSS_REFERENCE
    N, D_in, bits, group = 256, 512, 4, 128
    D_fit = _largest_fitting_d_out(awq, N, D_in, 21, bits, group, fid)
    assert awq.search_workspace_size(N, D_in, D_fit, 21, bits, group, fid) <= SCRATCH_BYTES
    need = awq.search_workspace_size(N, D_in, D_fit + 4, 21, bits, group, fid)
    assert need > SCRATCH_BYTES
    _check_against_workspace_search(awq, fn, N, D_in, D_fit, bits, group, fid, seed=11)
    X = torch.zeros(N, D_in, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(D_in, D_fit + 4, dtype=torch.float32, device="cuda")
    a = torch.ones(D_in, dtype=torch.float32, device="cuda")
    out = torch.empty(64, dtype=torch.float64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = _call(fn, X, W, a, synth.alpha_grid(20).tolist(), bits, group, fid, out, None, out, out, status)
    assert rc == AWQ_EWORKSPACE
    msg = awq.last_error()
    assert str(need) in msg and str(SCRATCH_BYTES) in msg


def test_noalloc_rejects_shapes_far_beyond_the_scratch(lib):
    awq, fn = lib
    # 4096 x 4096 with 21 alphas needs far more than the built-in scratch.
    N, D_in, D_out = 4096, 4096, 4096
    need = awq.search_workspace_size(N, D_in, D_out, 21, 4, 128)
    assert need > SCRATCH_BYTES
    X = torch.zeros(16, D_in, dtype=torch.bfloat16, device="cuda")     # never read: rejected first
    W = torch.zeros(16, D_out, dtype=torch.float32, device="cuda")
    a = torch.ones(D_in, dtype=torch.float32, device="cuda")
    out = torch.empty(64, dtype=torch.float64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = (ctypes.c_float * 21)(*synth.alpha_grid(20).tolist())
    rc = fn(X.data_ptr(), W.data_ptr(), a.data_ptr(), N, D_in, D_out, g, 21, 4, 128, 0, out.data_ptr(), None,
            out.data_ptr(), out.data_ptr(), status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == AWQ_EWORKSPACE
    msg = awq.last_error()
    assert str(need) in msg and str(SCRATCH_BYTES) in msg


def test_noalloc_requires_a_status_word(lib):
    """Without the caller's status word a device-side timeout could not be
    seen, so the call refuses a NULL status before any work."""
    awq, fn = lib
    X = torch.zeros(256, 512, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(512, 512, dtype=torch.float32, device="cuda")
    a = torch.ones(512, dtype=torch.float32, device="cuda")
    out = torch.empty(64, dtype=torch.float64, device="cuda")
    rc = _call(fn, X, W, a, synth.alpha_grid(20).tolist(), 4, 128, 0, out, None, out, out, None)
    assert rc == AWQ_EINVAL
    assert "status" in awq.last_error()
