"""The microbenchmarks of the forward's MMA issue compile for sm_100a (nvcc
cross-compiles without a GPU); running them needs a B200."""

import os

import pytest

from exact_softmax_attention_02_b200 import microbench


@pytest.mark.parametrize("name", microbench.PROGRAMS)
def test_microbenchmark_builds(name):
    path = microbench.build(name)
    assert os.path.isfile(path) and os.access(path, os.X_OK)


def test_unknown_microbenchmark_is_rejected():
    with pytest.raises(SystemExit):
        microbench.main(["nonsense"])
