"""Device-side failure detection without a GPU fault.

Every wait of the pipeline kernels is bounded: when one runs out, the kernel
records CSA_ERR_TIMEOUT in the device error word, lets what it issued land and
returns, and csa_get_error reports it. Here one bounded wait is made to run
out on purpose (a barrier that nothing completes, csa_debug_wait_probe) and
the test checks that the status reaches the host, that reading it clears it,
and that the device still runs the path correctly afterwards.
"""
import math

import numpy as np
import pytest
import torch

from long_context_sparse_07_b200 import abi, path, workloads as W

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_device_stays_usable():
    abi.load()
    abi.csa_get_error()
    abi.csa_debug_wait_probe(1_000_000)          # 1 ms, then give up
    with pytest.raises(abi.CsaError) as ei:
        abi.csa_get_error()
    assert ei.value.status == -4
    assert "timed out" in str(ei.value) and "kernel 8" in str(ei.value)
    # the word was cleared by the read
    assert abi.csa_get_error() == 0
    # a normal step still runs and the error word stays clear
    w = W.scaled(W.WORKLOADS["csa_bf16_n4096"], n=512)
    p = path.CsaPrefill(w, W.csa_operands(w))
    p.step()
    assert abi.csa_get_error() == 0
    assert torch.isfinite(p.out.float()).all()
    # twice in a row, on another stream
    s = torch.cuda.Stream()
    abi.csa_debug_wait_probe(2_000_000, stream=s)
    abi.csa_debug_wait_probe(1_000_000, stream=s)
    with pytest.raises(abi.CsaError) as ei:
        abi.csa_get_error()
    assert ei.value.status == -4
    assert abi.csa_get_error() == 0
