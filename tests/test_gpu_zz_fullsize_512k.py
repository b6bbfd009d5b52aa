"""Parity at the 512K workload (B=1, T=524288, Hq=16, Hkv=4, d=128, dp=64,
topk=128), with the same sampled checks, whole-tensor identities and
masked-dO shared-block checks as the 32K and 128K cases, in the benchmark's
launch configuration.  Kept in its own
file, run after the others: it is the longest case (about a minute of oracle
work on the host)."""
import pytest

import test_gpu_fullsize as fullsize

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_full_size_512k():
    fullsize.test_full_size("512k", 128, 256, 384)
