"""The device-side error path without a fault: a bounded wait with a short limit runs out on a barrier
nothing arrives on, the kernel records the device error word and returns, csa_device_status reports
CSA_ERR_DEVICE once (and clears it), and the context stays usable for the layer's own kernels."""
import ctypes

import pytest
import torch

from csa_workloads import gen, normal

pytestmark = pytest.mark.gpu
DEV = "cuda"
CSA_OK, CSA_ERR_INVALID, CSA_ERR_DEVICE = 0, 1, 5


def test_bounded_wait_timeout_is_reported_and_cleared(cuda_lib):
    csa = cuda_lib
    lib = csa._lib
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.csa_device_status(ctypes.c_void_p(stream)) == CSA_OK          # nothing recorded yet
    assert lib.csa_check_error_path(0, ctypes.c_void_p(stream)) == CSA_ERR_INVALID
    assert lib.csa_check_error_path(1000, ctypes.c_void_p(stream)) == CSA_OK  # launched; the wait gives up
    assert lib.csa_device_status(ctypes.c_void_p(stream)) == CSA_ERR_DEVICE
    assert lib.csa_device_status(ctypes.c_void_p(stream)) == CSA_OK          # read and cleared
    # the Python binding raises on the recorded error
    csa.check_error_path(200)
    with pytest.raises(csa.CSAError, match="CSA_ERR_DEVICE"):
        csa.device_status()
    csa.device_status()


def test_context_usable_after_the_error_path(cuda_lib):
    """After a recorded timeout the same process runs the indexer + top-k and the status is clean."""
    csa = cuda_lib
    csa.check_error_path(500)
    with pytest.raises(csa.CSAError):
        csa.device_status()
    G = gen(5, DEV)
    B, n, k = 2, 3000, 64
    ki = csa.PackedCache(B, n, 128, 0, DEV)
    csa.pack_fp4(normal((B, n, 128), 1.0, G, DEV), ki)
    qI = normal((B, 1, 8, 128), 1.0, G, DEV)
    w = normal((B, 1, 8), 0.35, G, DEV, torch.float32)
    n_c = torch.full((B,), n, dtype=torch.int32, device=DEV)
    q_pos = torch.full((B, 1), 4 * n - 1, dtype=torch.int64, device=DEV)
    idx, _, _ = csa.index_topk(qI, w, ki, n_c, q_pos, ratio=4, k=k)
    csa.device_status()
    assert int((idx >= 0).sum()) == B * k
