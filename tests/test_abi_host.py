"""Host-side checks of the C-ABI library (no GPU needed, no compute call).

The library must build for sm_100a, load, export every function that
include/csa.h declares, and reject bad arguments during host validation,
before it touches the CUDA runtime.
"""
import ctypes
import os
import re

import pytest
import torch

from long_context_sparse_07_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    txt = open(os.path.join(ROOT, "include", "csa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", txt, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert "csa_compress_kv" in names and "hca_dense_mqa" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(abi.EXPORTS) | set(names)
    assert set(abi.EXPORTS) <= set(names)


def test_version_and_status_strings(lib):
    assert lib.csa_abi_version() == 1
    assert lib.csa_status_string(-5) == b"index out of bounds on the device"
    assert lib.csa_status_string(0) == b"ok"


def _entries(body=0x1000, c=64, dt=abi.CSA_BF16, **kw):
    e = abi._Entries(body, kw.get("scale"), kw.get("rope"), c, kw.get("rope_dims", 0),
                     kw.get("scale_group", 0), dt)
    return e


def test_compress_rejects_bad_arguments_before_any_launch(lib):
    P = 0x10000
    # missing Ca
    st = lib.csa_compress_kv(None, P, P, P, P, P, 16, 64, 4, 1, abi.CSA_BF16, _entries(), None)
    assert st == -1 and b"required" in lib.csa_last_message()
    # n not a multiple of m
    st = lib.csa_compress_kv(P, P, P, P, P, P, 18, 64, 4, 1, abi.CSA_BF16, _entries(), None)
    assert st == -1 and b"multiple of m" in lib.csa_last_message()
    # misaligned input
    st = lib.csa_compress_kv(P + 2, P, P, P, P, P, 16, 64, 4, 1, abi.CSA_BF16, _entries(), None)
    assert st == -1 and b"aligned" in lib.csa_last_message()
    # no overlap but a second window given
    st = lib.csa_compress_kv(P, P, P, P, P, P, 16, 64, 4, 0, abi.CSA_BF16, _entries(), None)
    assert st == -1
    # unsupported width
    st = lib.csa_compress_kv(P, P, P, P, P, P, 16, 72, 4, 1, abi.CSA_BF16, _entries(c=72), None)
    assert st == -2
    # fp8 output without scales
    st = lib.csa_compress_kv(P, P, P, P, P, P, 16, 64, 4, 1, abi.CSA_BF16,
                             _entries(dt=abi.CSA_E4M3, scale_group=64), None)
    assert st == -1 and b"scales" in lib.csa_last_message()


def test_indexer_topk_attend_reject_bad_arguments(lib):
    P = 0x10000
    k = _entries(c=128)
    st = lib.csa_indexer_scores(P, None, P, k, P, 1, 10, 10, 4, 128, 4, abi.CSA_E4M3, P, 10,
                                None)
    assert st == -1          # key dtype differs from query dtype
    st = lib.csa_indexer_scores(P, None, P, k, P, 1, 10, 10, 300, 128, 4, abi.CSA_BF16, P, 10,
                                None)
    assert st == -2          # too many heads
    st = lib.csa_indexer_scores(P, None, P, k, P, 1, 10, 10, 4, 128, 4, abi.CSA_BF16, P, 5, None)
    assert st == -1          # ld < E
    assert lib.csa_topk(P, 4, 10, 10, P, 4, 0, P, None, 0, None) == -2          # k = 0
    assert lib.csa_topk(None, 4, 10, 10, P, 4, 3, P, None, 0, None) == -1
    kv = _entries(c=512)
    st = lib.csa_sparse_mqa(P, abi.CSA_BF16, kv, 10, 4, None, 5, P, 10, None, 4, P, P, 1, 4,
                            8, 0.1, P, None, None, 0, None)
    assert st == -1 and b"idx" in lib.csa_last_message()
    st = lib.hca_dense_mqa(P, abi.CSA_F32, _entries(c=512, dt=abi.CSA_E4M3, scale=P,
                                                     scale_group=64), 10, 128, P, 10, None, 4,
                           P, P, 1, 4, 8, 0.1, P, None, None, 0, None)
    assert st == -2          # fp8 entries need bf16 queries
    st = lib.hca_dense_mqa(P, abi.CSA_BF16, _entries(c=96), 10, 128, P, 10, None, 4, P, P, 1,
                           4, 8, 0.1, P, None, None, 0, None)
    assert st == -2          # c not a multiple of 64


def test_product_path_does_not_touch_the_oracle():
    pkg = os.path.join(ROOT, "long_context_sparse_07_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "csa_oracle" not in src, f


def test_wait_probe_rejects_limits_outside_its_range(lib):
    assert lib.csa_debug_wait_probe(10, None) == -1
    assert b"limit_ns" in lib.csa_last_message()
    assert lib.csa_debug_wait_probe(5 * 10 ** 9, None) == -1


def test_no_alloc_validates_before_touching_the_device(lib):
    P = 0x10000
    kv = _entries(c=512)
    st = lib.csa_sparse_mqa_noalloc(P, abi.CSA_BF16, kv, 10, 4, None, 5, P, 10, None, 4, P, P, 1,
                                    4, 8, 0.1, P, None, None)
    assert st == -1 and b"idx" in lib.csa_last_message()


def test_topk_workspace_contract(lib):
    # rows up to 2048 .. 64 K entries and rows of 64 K .. 256 K entries (one
    # cluster of blocks per row) need no workspace; longer rows are split over
    # many blocks in four launches and need one that grows with rows * E
    for E in (1024, 40000, 65535, 65536, 100000, 262144):
        assert abi.csa_topk_workspace_size(8, E, 1024) == 0, E
    small = abi.csa_topk_workspace_size(2, 300000, 1024)
    assert small >= 2 * 300000 * 16
    assert abi.csa_topk_workspace_size(4, 300000, 1024) > small
    # decode through the one-call entry: the indexer, then one top-k launch
    assert abi.csa_indexer_topk_launches(8, 1, 262144, 64, 128, 1024, abi.CSA_E4M3) == 2
    assert abi.csa_indexer_topk_launches(2, 1, 300000, 64, 128, 1024, abi.CSA_E4M3) == 5
