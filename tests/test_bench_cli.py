"""bench.py's command line on a host without a GPU: argument checks and the
experiments' refusal to run without a CUDA device (none of them falls back to
the CPU)."""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=300, cwd=ROOT)


@pytest.fixture(scope="module")
def no_cuda():
    import torch

    if torch.cuda.is_available():
        pytest.skip("this host has a GPU; the experiments are covered by the GPU tests")


def test_warmup_below_three_is_rejected():
    r = _bench("--warmup", "2", "--steps", "1")
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr


def test_unknown_experiment_is_rejected():
    r = _bench("--experiment", "nonsense")
    assert r.returncode != 0
    assert "invalid choice" in r.stderr


@pytest.mark.parametrize("experiment", ["sparse", "tiles"])
def test_experiments_need_a_cuda_device(no_cuda, experiment):
    r = _bench("--experiment", experiment, "--steps", "3")
    assert r.returncode != 0
    assert "needs a CUDA device" in (r.stderr + r.stdout)
    # no JSON line is printed in place of a measurement
    assert not r.stdout.strip().startswith("{")
