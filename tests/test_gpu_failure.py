"""The failure path of the bounded device-side waits, on the GPU and without a
fault: a wait on a barrier that nothing sets gives up after its limit, the host
reads SAS_ERR_DEVICE_TIMEOUT from the device status word once, and the context
stays usable for the next call."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable(cuda_ok):
    from trainable_block_sparse_sas_b200 import api

    api.sas_device_status()  # clean start
    api.sas_selftest_bounded_wait(50)
    with pytest.raises(api.SasError) as e:
        api.sas_device_status()
    assert e.value.status == api.SAS_ERR_DEVICE_TIMEOUT
    api.sas_device_status()  # reported once, then cleared
    # the context still runs kernels correctly
    s = torch.tensor([[[[0.8, 1.5, 0.3, 0.6, 0.0]]]], device="cuda")
    idx = torch.empty((1, 1, 1, 2), dtype=torch.int32, device="cuda")
    api.sas_topk_select(s, 1, 5, 2, idx=idx, ctx_len=torch.tensor([5 * 64 + 1], dtype=torch.int32, device="cuda"),
                        block_size=64)
    torch.cuda.synchronize()
    assert idx.cpu().numpy().ravel().tolist() == [0, 1]


def test_selftest_rejects_bad_limits(cuda_ok):
    from trainable_block_sparse_sas_b200 import api

    for bad in (0, -5, 20000):
        with pytest.raises(api.SasError) as e:
            api.sas_selftest_bounded_wait(bad)
        assert e.value.status == api.SAS_ERR_INVALID_VALUE
