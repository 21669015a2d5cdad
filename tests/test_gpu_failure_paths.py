"""Failure paths surface as status codes, without faulting, trapping or
hanging the GPU: a device-side wait that runs out is reported as
MOE_ERR_TIMEOUT and leaves the context usable; a failed scratch allocation
makes moe_layer_create return MOE_ERR_OOM and leaks nothing."""
import pytest

import synth
from helpers import bf16_close
from gpu_common import create_layer, make_device_layer, oracle_layer_for, residual_tokens, to_host_u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from sparse_moe_decode_router_b200 import api
    api.load_library()
    return torch


def _tiny_forward_matches_oracle(torch, dl):
    from sparse_moe_decode_router_b200 import api
    x_h, x_d = dl.tokens([3])
    r_h, r_d = residual_tokens(dl.cfg, [3])
    h = create_layer(dl, 1)
    try:
        out = torch.empty((1, dl.cfg.hidden), dtype=torch.bfloat16, device="cuda")
        api.moe_layer_forward(h, None, x_d, r_d, out, 1)
        torch.cuda.synchronize()
        assert api.moe_layer_last_device_error(h) == api.MOE_OK
        ok, info = bf16_close(to_host_u16(out), oracle_layer_for(dl, x_h, r_h)["out_bf16"])
        assert ok, info
    finally:
        api.moe_layer_destroy(h)


def test_device_wait_timeout_is_reported(torch_cuda):
    from sparse_moe_decode_router_b200 import api
    assert api.moe_selftest(api.MOE_SELFTEST_WAIT_TIMEOUT) == api.MOE_ERR_TIMEOUT
    # the context is still usable afterwards
    _tiny_forward_matches_oracle(torch_cuda, make_device_layer(synth.CONFIGS[0]))


def test_injected_allocation_failure(torch_cuda):
    from sparse_moe_decode_router_b200 import api
    dl = make_device_layer(synth.CONFIGS[0])
    free0 = torch_cuda.cuda.mem_get_info()[0]
    assert api.moe_selftest(api.MOE_SELFTEST_FAIL_NEXT_ALLOC) == api.MOE_OK
    with pytest.raises(api.MoEError) as e:
        create_layer(dl, 4)
    assert e.value.status == api.MOE_ERR_OOM
    assert torch_cuda.cuda.mem_get_info()[0] >= free0 - (8 << 20)  # nothing of note left allocated
    # one-shot: the next layer is created and works
    _tiny_forward_matches_oracle(torch_cuda, dl)
