"""The allocation-free decode entry point, for callers that cannot allocate
device memory (a serving engine whose memory is all in its own pool, or code
inside a CUDA graph capture). It must give the same result as paro_linear,
within the parity tolerances the other tests use, on two calls in a row
(the static scratch keeps the previous call's contents). Collected last on
purpose."""
import ctypes

import numpy as np
import pytest
import torch

import synth

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
    for call, T in enumerate((16, 5)):                   # two calls in a row, different batches
        X = torch.from_numpy(synth.activations(T, n_in, seed + call)).cuda()
        ref = B.paro_linear(rot, X, qw, sp, zp, n_out)
        Y = torch.full((T, n_out), float("nan"), dtype=torch.float16, device="cuda")
        st = L.paro_linear_noalloc(rot.handle, X.data_ptr(), qw.data_ptr(), sp.data_ptr(), zp.data_ptr(),
                                   Y.data_ptr(), T, n_in, n_out, stream)
        assert st == 0, L.paro_last_error()
        torch.cuda.synchronize()
        a, b = Y.double().cpu().numpy(), ref.double().cpu().numpy()
        assert np.all(np.isfinite(a))
        # the parity tolerance: Frobenius 2e-3; per element 1e-2, or one fp16
        # ulp plus 2e-3 where an ulp exceeds that (|Y| >= 16: either neighbour)
        rel = np.linalg.norm(a - b) / np.linalg.norm(b)
        ulp = np.abs(np.spacing(np.abs(b).astype(np.float16))).astype(np.float64)
        worst = np.max(np.abs(a - b) - np.maximum(1e-2, ulp + 2e-3))
        assert rel <= 2e-3 and worst <= 0.0, (rel, np.max(np.abs(a - b)))


def test_noalloc_rejects_oversize(cuda_lib):
    from rotated_w4_linear_b200 import binding as B
    L = B.lib()
    # 17 tokens, and 16 tokens x 65536 channels (2 MiB > 1 MiB of static scratch)
    assert L.paro_linear_noalloc(None, None, None, None, None, None, 17, 4096, 1024, None) == 1
    assert L.paro_linear_noalloc(None, None, None, None, None, None, 16, 65536, 1024, None) == 1
    assert b"static scratch" in L.paro_last_error()
