"""Router and shared-expert variants the pages leave open, through the C ABI
against the oracle: the bias-corrected sigmoid router (scores
sigmoid(logit), selection by score + bias, weights normalised scores) and a
shared expert stored in MXFP4 like the routed ones.  Each runs on the
CUDA-core expert kernels, the grouped kernels (batch > 8) and the tcgen05
kernels."""
import pytest

import synth
from gpu_common import make_device_layer
from test_gpu_parity import check_against_oracle, run_all_paths

pytestmark = pytest.mark.gpu

SIGMOID = 0x20
MX = 0x10
CUDA_CORES = 0x8  # MOE_FLAG_NO_GROUPED: the GEMVs at every batch size


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from sparse_moe_decode_router_b200 import api
    api.load_library()
    return torch


@pytest.fixture(scope="module")
def sigmoid_layer(torch_cuda):
    base = synth.CONFIGS[0]
    cfg = base.with_(hidden=512, inter=256, shared_inter=64, zipf_s=0.2, scoring="sigmoid", seed=base.seed + 500)
    return make_device_layer(cfg)


@pytest.fixture(scope="module")
def shared_mx_layer(torch_cuda):
    base = synth.CONFIGS[0]
    cfg = base.with_(hidden=512, inter=256, shared_inter=128, shared_format="mxfp4", seed=base.seed + 600)
    return make_device_layer(cfg)


@pytest.mark.parametrize("flags", [CUDA_CORES, MX], ids=["cuda_cores", "tcgen05"])
@pytest.mark.parametrize("B", [1, 5, 33])
def test_sigmoid_router_matches_oracle(torch_cuda, sigmoid_layer, B, flags):
    got, ref = run_all_paths(torch_cuda, sigmoid_layer, B, max_batch=64, flags=SIGMOID | flags)
    check_against_oracle(got, ref)


@pytest.mark.parametrize("flags", [CUDA_CORES, MX], ids=["cuda_cores", "tcgen05"])
@pytest.mark.parametrize("B", [1, 5, 33])
def test_mxfp4_shared_expert_matches_oracle(torch_cuda, shared_mx_layer, B, flags):
    got, ref = run_all_paths(torch_cuda, shared_mx_layer, B, max_batch=64, flags=flags)
    check_against_oracle(got, ref, shared_mx=True)


def test_full_size_sigmoid_router_and_mxfp4_shared_expert(torch_cuda):
    """Full-size layer, batch 1, both variants together (router weights at a
    smaller scale so that sigmoid scores keep a decision margin)."""
    cfg = synth.CONFIGS[1].with_(scoring="sigmoid", zipf_s=0.2, router_sigma=0.01, shared_format="mxfp4",
                                 seed=synth.CONFIGS[1].seed + 700)
    dl = make_device_layer(cfg)
    try:
        got, ref = run_all_paths(torch_cuda, dl, 1, flags=SIGMOID)
        check_against_oracle(got, ref, shared_mx=True)
    finally:
        del dl
        torch_cuda.cuda.empty_cache()
