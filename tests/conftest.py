import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(params=[1, 2, 3], ids=["1tile", "2tiles", "keysplit"])
def prefill_tiles(request):
    """Run the test with the one-tile tcgen05 prefill kernel, the two-tile
    kernel on pairs of query tiles, and the two-tile kernel with one query
    tile's key range split between its softmax warpgroups (pinned through
    the library's test hook, released afterwards)."""
    import rotary_embedding_b200 as fa
    fa.fa_testing_set_prefill_tiles(request.param)
    yield request.param
    fa.fa_testing_set_prefill_tiles(0)
