"""Host logic of the pipelined step from host buffers: the query chunk
schedule covers every query once, in order, with no chunk above the
requested size, small chunks first and last when there is room for them."""
import pytest

from long_context_sparse_07_b200.path import CsaPrefill


@pytest.mark.parametrize("nq,chunk", [(131072, 16384), (65536, 16384), (61440, 16384),
                                      (40000, 16384), (16384, 16384), (4096, 1000), (1, 16384),
                                      (131072, 2048), (100000, 8192)])
def test_chunk_plan_partitions_the_queries(nq, chunk):
    plan = CsaPrefill.chunk_plan(nq, chunk)
    assert sum(plan) == nq and all(0 < r <= chunk for r in plan)


def test_chunk_plan_ramps_at_both_ends():
    plan = CsaPrefill.chunk_plan(131072, 16384)
    assert plan[:3] == [2048, 4096, 8192] and plan[-3:] == [8192, 4096, 2048]
    assert plan.count(16384) == 6
    # too few queries for both ramps: plain chunks
    assert CsaPrefill.chunk_plan(40000, 16384) == [16384, 16384, 7232]
