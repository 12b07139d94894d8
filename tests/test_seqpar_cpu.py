"""Sequence parallelism on CPU: one CSA prefill split over two gloo ranks.

Each rank owns two zig-zag token chunks, receives the rows before them (the
compression and window halos) through one all-gather of chunk tails,
compresses its chunks, all-gathers the compressed entries and indexer keys,
and runs the indexer, top-k and attention of its own queries. The per-rank
steps run on a CPU stand-in built from the oracle (on a GPU the same host
logic calls the C ABI); the outputs of all ranks, put back in sequence order,
must equal the oracle's single-rank chain.
"""
import math
import os
import pickle
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import oracle  # noqa: E402
from oracle import pipeline  # noqa: E402
from long_context_sparse_07_b200 import seqpar, workloads as W  # noqa: E402


class OracleBackend:
    """The four per-rank steps on the CPU, from the oracle, storing each
    result in the path's storage dtype (as the GPU calls do)."""

    def compress(self, kind, xs, Ba, Bb, w):
        Ca, Cb, Za, Zb = xs
        e64 = oracle.compress(Ca, Cb, Za, Zb, Ba, Bb, w.m, True)
        if kind == "ki" and w.idx_dtype == "e4m3":
            codes, scales = oracle.quantize_e4m3(e64, w.cI)
            return (torch.from_numpy(codes).view(torch.float8_e4m3fn),
                    torch.from_numpy(scales[:, 0].copy()))
        dt = w.dtype if kind == "kv" else w.idx_dtype
        st = pipeline.store(e64, dt)
        t = torch.from_numpy(st).to(torch.float32)
        return (t.to(torch.bfloat16) if dt == "bf16" else t, None)

    def _values(self, body, scale, width):
        if scale is not None:
            return oracle.dequantize(body, scale.view(-1, 1), width)
        return oracle.f64(body)

    def indexer(self, loc, ki, pos, w):
        if w.idx_dtype == "e4m3":
            qI = oracle.dequantize(loc["qI"], loc["qI_scale"].reshape(-1, w.hI, 1), w.cI)
        else:
            qI = oracle.f64(loc["qI"])
        kI = self._values(ki[0], ki[1], w.cI)
        sc = oracle.indexer(qI[None], oracle.f64(loc["wI"])[None], kI[None],
                            pos.numpy()[None], w.m)[0]
        return torch.from_numpy(sc.astype(np.float32))

    def topk(self, sc, pos, w):
        return torch.from_numpy(oracle.topk(sc.double().numpy(), pos.numpy(), w.m, w.k))

    def attend(self, q, ent, idx, kwin, win_pos0, pos, sink, w):
        out, lse = oracle.attend(oracle.f64(q)[None], oracle.f64(ent[0])[None], idx.numpy(),
                                 w.k, w.m, oracle.f64(kwin)[None], [win_pos0], w.n_win,
                                 pos.numpy()[None], sink, 1.0 / math.sqrt(w.c))
        return torch.from_numpy(out[0]), torch.from_numpy(lse[0])


WORKLOADS = {
    "fp32": W.scaled(W.WORKLOADS["csa_fp32_n256"], n=256),
    "bf16_e4m3": W.scaled(W.WORKLOADS["csa_fp8idx_n131072"], n=384, c=64, hI=4, cI=32, k=16,
                          n_win=24, h=4, name="small_fp8idx"),
}


def _rank_main(rank, world, port, name, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS[name]
        ops = W.csa_operands(w)
        sp = seqpar.SeqParallelCsa(w, OracleBackend(), dist)
        local = sp.local_operands(ops)
        shared = {k: ops[k] for k in ("Ba", "Bb", "BIa", "BIb", "sink")}
        res = sp.run(local, shared)
        with open(os.path.join(out_dir, "r%d.pkl" % rank), "wb") as f:
            pickle.dump({j: tuple(x.numpy() for x in v) for j, v in res.items()}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_two_ranks_reproduce_the_single_rank_chain(tmp_path, name):
    world = 2
    port = 29600 + (os.getpid() % 500) + (7 if name == "fp32" else 0)
    mp.start_processes(_rank_main, args=(world, port, name, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    w = WORKLOADS[name]
    ref = pipeline.csa_prefill(W.csa_operands(w), w)
    got_out = np.full(ref["out"].shape, np.nan)
    got_lse = np.full(ref["lse"].shape, np.nan)
    got_idx = np.full(ref["idx"].shape, -9, dtype=np.int64)
    seen = 0
    for r in range(world):
        with open(tmp_path / ("r%d.pkl" % r), "rb") as f:
            part = pickle.load(f)
        for j, (pos, out, lse, idx) in part.items():
            got_out[pos], got_lse[pos], got_idx[pos] = out, lse, idx
            seen += len(pos)
    assert seen == w.n
    np.testing.assert_array_equal(got_idx, ref["idx"])
    np.testing.assert_allclose(got_out, ref["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_lse, ref["lse"], rtol=0, atol=1e-12)


def test_chunks_cover_the_sequence_in_whole_blocks():
    for n, m, P in ((256, 4, 2), (384, 4, 3), (1000, 8, 4), (64, 4, 8)):
        ch = seqpar.chunks(n, m, P)
        assert ch[0][0] == 0 and ch[-1][1] == (n // m) * m
        assert all(a % m == 0 and b % m == 0 and a <= b for a, b in ch)
        assert all(ch[i][1] == ch[i + 1][0] for i in range(len(ch) - 1))
        got = sorted(j for r in range(P) for j in seqpar.owned(P, r))
        assert got == list(range(2 * P))
