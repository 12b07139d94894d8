"""The prefill step from pinned host operands to a pinned host output, with the
copies overlapped with the computation (queries in chunks), gives exactly the
device-resident step's output and lse."""
import pytest
import torch

from long_context_sparse_07_b200 import abi, path, workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,n,chunk", [
    ("csa_bf16_n4096", None, 1000),            # the two plain calls inside, a ragged last chunk
    ("csa_fp8idx_n131072", 65536, 16384),      # the one-call candidate path per chunk
    ("csa_fp8idx_n131072", 65536, 8192),       # chunks ramping 2048 -> 8192 -> 2048
])
def test_step_from_host_equals_device_step(name, n, chunk):
    w = W.WORKLOADS[name]
    if n is not None:
        w = W.scaled(w, n=n, name="%s@n%d" % (name, n))
    ops = W.csa_operands(w)
    p = path.CsaPrefill(w, ops, fused=True)
    if name == "csa_fp8idx_n131072" and chunk == 16384:
        assert abi.csa_indexer_topk_launches(1, chunk, w.E, w.hI, w.cI, w.k, p.d["qI"]) == 6
    p.step()
    torch.cuda.synchronize()
    abi.csa_get_error()
    ref_out, ref_lse = p.out.clone(), p.lse.clone()
    host_in = {k: v.cpu().pin_memory() for k, v in p.inputs().items()}
    for v in p.inputs().values():                 # the device copies must come from the host
        v.zero_()
    p.out.zero_()
    p.lse.zero_()
    host_out = torch.empty(p.out.shape, dtype=p.out.dtype, pin_memory=True)
    p.step_from_host(host_in, host_out, chunk=chunk)
    torch.cuda.synchronize()
    abi.csa_get_error()
    assert torch.equal(host_out, ref_out.cpu())
    assert torch.equal(p.lse, ref_lse)
