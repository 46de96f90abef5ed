"""The allocation-free decode entry point, paro_linear_noalloc.

It serves callers that cannot allocate device memory: a serving engine that
hands all device memory to its own pool at start-up, or code that must not
call cudaMalloc while a CUDA graph is being captured. It runs the same
kernels with the same plan as paro_linear, only with its X T^-1 scratch in a
static device array. Its output must agree with paro_linear's within the
parity tolerances the other tests use, on two calls in a row (the array keeps
the previous call's contents, here from a larger batch, which must not leak
into the next); both calls are also checked against the CPU fp64 oracle.
(The decode kernel adds warp partial sums with shared-memory atomics, whose
order varies from run to run, so two calls may differ in the last bit.)
Collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import synth
from oracle import paro_oracle as O  # noqa: F401  (used through parity.check_linear)
from parity import check_linear, output_bound

pytestmark = pytest.mark.gpu


def test_noalloc_matches_paro_linear_twice(cuda_lib):
    from rotated_w4_linear_b200 import binding as B
    L = B.lib()
    n_in, n_out, K = 4096, 1024, 8
    seed = synth.layer_seed(2, 77)
    pairs, theta, alpha = synth.rotation_params(n_in, K, seed)
    q, s, z = synth.w4_codes(n_out, n_in, seed)
    qw, sp, zp = B.paro_pack_weights(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(),
                                     torch.from_numpy(z).cuda())
    rot = B.paro_rot_create(pairs, theta, alpha)
    stream = torch.cuda.current_stream().cuda_stream
    for call, T in enumerate((16, 5)):                   # two calls in a row, the second smaller
        x = synth.activations(T, n_in, seed + call)
        X = torch.from_numpy(x).cuda()
        ref = B.paro_linear(rot, X, qw, sp, zp, n_out)
        Y = torch.full((T, n_out), float("nan"), dtype=torch.float16, device="cuda")
        st = L.paro_linear_noalloc(rot.handle, X.data_ptr(), qw.data_ptr(), sp.data_ptr(), zp.data_ptr(),
                                   Y.data_ptr(), T, n_in, n_out, stream)
        assert st == 0, L.paro_last_error()
        torch.cuda.synchronize()
        got, want = Y.cpu().numpy(), ref.cpu().numpy()
        a, b = got.astype(np.float64), want.astype(np.float64)
        assert np.all(np.isfinite(a))
        assert np.linalg.norm(a - b) <= 2e-3 * np.linalg.norm(b), call
        assert np.all(np.abs(a - b) <= output_bound(a, b, b)), call
        check_linear(got, x, pairs, theta, alpha, q, s, z)
    assert B.paro_fault_status() == 0


def test_noalloc_rejects_oversize(cuda_lib):
    from rotated_w4_linear_b200 import binding as B
    L = B.lib()
    # 17 tokens, and 16 tokens x 65536 channels (2 MiB > 1 MiB of static scratch)
    assert L.paro_linear_noalloc(None, None, None, None, None, None, 17, 4096, 1024, None) == 1
    assert L.paro_linear_noalloc(None, None, None, None, None, None, 16, 65536, 1024, None) == 1
    assert b"static scratch" in L.paro_last_error()
