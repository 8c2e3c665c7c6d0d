import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes of oracle time)")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=[1, 2], ids=["tile256", "tile512"])
def gemm_tile(request):
    """Runs a GPU test once with each GEMM pair tile (256 x 256 and 256 x 512)."""
    import rl_post_policy_b200 as pl
    assert pl.pl_debug_set_gemm_tile(request.param) == 0
    yield request.param
    pl.pl_debug_set_gemm_tile(0)


@pytest.fixture(params=[(1, 0, 0), (2, 1, 2), (1, 2, 0)], ids=["merged", "separate_ksplit_fused_finish",
                                                                 "merged_ew4"])
def gemm_variant(request):
    """Runs a GPU test with each way the fused path may launch its GEMMs: several
    chunks' backward and next forward merged into one dynamically scheduled launch,
    with a separate pass rounding the fp32 dW accumulator (the default); separate
    launches with the backward's dX problem split in two K halves and the last
    chunk's dW epilogue finishing the fp32 accumulation; and merged launches with
    4 epilogue warps."""
    import rl_post_policy_b200 as pl
    split, merge, finish = request.param
    assert pl.pl_debug_set_gemm_split(split) == 0
    assert pl.pl_debug_set_gemm_merge(merge) == 0
    assert pl.pl_debug_set_dw_finish(finish) == 0
    yield request.param
    pl.pl_debug_set_gemm_split(0)
    pl.pl_debug_set_gemm_merge(0)
    pl.pl_debug_set_dw_finish(0)


@pytest.fixture(params=[1, 2], ids=["rkl_streaming", "rkl_resident"])
def rkl_path(request):
    """Runs a GPU test once with the streaming reverse-KL kernel and once with the
    register-resident gradient kernel wherever it applies."""
    import rl_post_policy_b200 as pl
    assert pl.pl_debug_set_rkl_path(request.param) == 0
    yield request.param
    pl.pl_debug_set_rkl_path(0)


@pytest.fixture(params=[1, 2], ids=["small_kernel", "cooperative"])
def loss_path(request):
    """Runs a GPU test once with each loss-only kernel: the small-batch kernel
    (used whenever the batch is small enough) and the cooperative kernel."""
    import rl_post_policy_b200 as pl
    assert pl.pl_debug_set_loss_path(request.param) == 0
    yield request.param
    pl.pl_debug_set_loss_path(0)
