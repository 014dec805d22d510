"""bench.py's algorithmic accounting on CPU: the per-kernel byte shares that
the dominant-kernel roofline divides by must add up to the path's bytes, and
the path's bytes and flops must follow their stated per-token-head forms."""
import dataclasses
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_deltanet_linear_chunked_b200 import workloads as wl  # noqa: E402

KERNELS = ("gdn_prep_kernel", "gdn_recur_kernel", "gdn_output_kernel")


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("dims", [(112, 112), (64, 128), (128, 32)])
def test_kernel_shares_sum_to_the_path(mode, dims):
    w = dataclasses.replace(wl.stream_chunk(mode), Dk=dims[0], Dv=dims[1])
    assert sum(bench.kernel_algorithmic_bytes(k, w) for k in KERNELS) == bench.algorithmic_bytes(w)


def test_path_bytes_of_the_streaming_chunk():
    # q, k, v, out in bf16 (2 bytes), g and beta in fp32, one fp32 state in
    # and one out per head: 2640 x 20 token-heads at d = 112
    w = wl.stream_chunk("fwd")
    token_heads = 2640 * 20
    expect = token_heads * (4 * 112 * 2 + 8) + 2 * 20 * 112 * 112 * 4
    assert bench.algorithmic_bytes(w) == expect


def test_path_flops_forms():
    w = wl.stream_chunk("fwd")
    d, c = 112, 64
    assert bench.algorithmic_flops(w) == 2640 * 20 * (6 * d * d + 8 * c * d)
    assert bench.algorithmic_flops(w, True) == 2 * bench.algorithmic_flops(w)
