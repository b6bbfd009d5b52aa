"""Parity at T = 1,048,576 (B=1, Hq=16, Hkv=4, d=128, dp=64, topk=128: the
512K workload's head shape at the top of the 512K -> 1M range), in the
benchmark's launch configuration: the selection of sampled queries bit for
bit, O, L and dQ of sampled rows, the whole-tensor identities, and fp32 dK/dV
of heavily shared blocks under a masked dO.  About 60 GB on the device; run
after every other GPU test file."""
import pytest

import test_gpu_fullsize as fullsize

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_full_size_1m():
    fullsize.test_full_size("1m", 64, 128, 128, last_blocks=False)
