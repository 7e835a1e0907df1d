"""GPU: the failure path of the kernels' bounded waits, exercised without a fault.

Every mbarrier wait in the library's kernels gives up after a wall-time limit, records
BSA_ERR_TIMEOUT and a site code in a device status word, and lets the kernel return.
`bsa_wait_timeout_selftest` runs that same wait on a barrier nothing ever arrives on;
the host must then read the time-out, the word must clear on read, and the context must
stay usable for real work.
"""

import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_tcgen05_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import block_sparse_attention_tcgen05_b200 as bsa
    from block_sparse_attention_tcgen05_b200 import _lib

    lib = _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    assert bsa.device_status()[0] == 0

    t0 = time.perf_counter()
    assert lib.bsa_wait_timeout_selftest(50_000_000, stream) == 0  # 50 ms
    st, where = bsa.device_status()
    elapsed = time.perf_counter() - t0
    assert st == _lib.BSA_ERR_TIMEOUT and where == 90, (st, where)
    assert 0.04 <= elapsed < 5.0, elapsed
    assert bsa.device_status() == (0, 0)  # cleared by the read

    # the context still runs real work correctly
    q, k, v = wl.gaussian_qkv(1, 1, 1, 256, 64, "bf16", seed=31)
    lab = np.arange(256) // 64
    mask = np.eye(4, dtype=bool)
    out = bsa.centroid_compensated_attention(
        q.to(dev), k.to(dev), v.to(dev), torch.as_tensor(lab, dtype=torch.int32, device=dev),
        torch.as_tensor(lab, dtype=torch.int32, device=dev),
        torch.as_tensor(mask, dtype=torch.uint8, device=dev), Cq=4, Ck=4)
    assert bsa.device_status()[0] == 0
    ref = oracle.centroid_compensated_attention(q.double().numpy(), k.double().numpy(),
                                                v.double().numpy(), lab, lab, mask)
    assert np.abs(out.cpu().numpy() - ref).max() <= 2e-2
