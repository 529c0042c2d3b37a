"""The tensor-parallel cases of tests/test_tp.py with the library's kernels as
the local products: two processes on cuda:0, collectives over gloo through host
memory (the ranks never wait on each other inside a kernel)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_two_rank_tensor_parallel_kernels_match_oracle(cuda_device):
    from test_tp import run_two_ranks
    run_two_ranks("cuda")
