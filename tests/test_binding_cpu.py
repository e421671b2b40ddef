"""The Python binding's own checks, which run before any C call: tensors that
are not on a CUDA device, or have the wrong dtype or shape, are refused with
ValueError (a host pointer or a short buffer handed to a kernel would be
read or written out of bounds on the device)."""
import pytest
import torch

from long_context_sequence_sca_b200 import lib as L

B, H, T, D = 1, 2, 256, 64


def _cpu(*shape, dtype=torch.float32):
    return torch.zeros(*shape, dtype=dtype)


@pytest.mark.parametrize("call", [
    lambda: L.sca_awm_forward(*[_cpu(B, H, T, D)] * 5, 128),
    lambda: L.sca_awm_forward_train(*[_cpu(B, H, T, D)] * 5, 128),
    lambda: L.sca_awm_forward_segment(*[_cpu(B, H, T, D)] * 5, 128),
    lambda: L.awm_segment_logsum(_cpu(B, H, T, D), 128),
    lambda: L.awm_segment_maps(_cpu(B, H, T, D), _cpu(B, H, T, D), _cpu(B, H, D), 128),
    lambda: L.awm_cp_logz(_cpu(2, B, H, D), 1),
    lambda: L.awm_cp_state(_cpu(2, B, H, D), _cpu(2, B, H, 4, D, D), 1),
    lambda: L.cema_forward(_cpu(B, T, D), *[_cpu(D, 16)] * 4, _cpu(D, 16, 2)),
    lambda: L.tdnorm_forward(_cpu(B, T, D), _cpu(D), _cpu(D), 8, 0.9, 0.99, 1e-5),
], ids=["forward", "forward_train", "segment", "segment_logsum", "segment_maps", "cp_logz", "cp_state",
        "cema", "tdnorm"])
def test_host_tensors_are_refused(call):
    with pytest.raises(ValueError):
        call()


def test_backward_refuses_host_tensors():
    x = [_cpu(B, H, T, D)] * 5
    with pytest.raises(ValueError):
        L.sca_awm_backward(*x, _cpu(B, H, T, D), _cpu(B, H, T), _cpu(B, H, T, D), _cpu(B, H, T, D), 128)
