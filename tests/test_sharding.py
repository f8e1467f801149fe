"""Sharding one problem over several devices or processes without exchanging
data (fa_shard_units, fa_shard_sequences and the sharded Python calls).

The forward's (batch, key/value head) units and decode's sequences are
independent problems: a query head reads only its own group's keys, a query
row only its own sequence's cache.  So a shard computes its own rows of o and
lse and the union of the shards is the result, with no collective on the data
path.  On the CPU: the partition helpers of libfa.so (which load without a
GPU), and two gloo ranks that each compute their shard with the fp64 oracle
and gather the pieces, which must equal the unsharded oracle bit for bit.  On
a GPU: the sharded calls over two shards of one device equal one launch.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from io_aware_exact_flashattention_b200 import build as fabuild
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import decode_inputs, prefill_inputs


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fabuild.build()
    fa.lib()


@pytest.mark.parametrize("B,Hkv,n", [(1, 1, 1), (2, 8, 3), (1, 8, 8), (3, 5, 7), (1, 2, 5),
                                     (64, 8, 4)])
def test_units_cover_every_unit_once_in_order(B, Hkv, n):
    ranges = [fa.shard_units(B, Hkv, n, s) for s in range(n)]
    pos = 0
    for first, count in ranges:
        assert first == pos and count >= 0
        pos += count
    assert pos == B * Hkv
    counts = [c for _, c in ranges]
    assert max(counts) - min(counts) <= 1


def test_units_reject_bad_arguments():
    for args in ((0, 1, 1, 0), (1, 0, 1, 0), (1, 1, 0, 0), (1, 1, 2, 2), (1, 1, 2, -1)):
        with pytest.raises(fa.FAError):
            fa.shard_units(*args)


@pytest.mark.parametrize("lens,n", [([5, 1, 1, 1, 100, 3], 3), ([1] * 10, 4), ([0, 0], 5),
                                    ([4096, 16384, 9000, 12000, 5000], 2), ([7], 1)])
def test_sequences_are_contiguous_and_balanced(lens, n):
    bounds = fa.shard_sequences(lens, n)
    assert len(bounds) == n + 1 and bounds[0] == 0 and bounds[-1] == len(lens)
    assert all(a <= b for a, b in zip(bounds, bounds[1:]))
    work = [max(L, 1) for L in lens]
    total = sum(work)
    prefix = np.concatenate([[0], np.cumsum(work)])
    for s in range(1, n):
        b = bounds[s]
        # smallest b' whose prefix holds at least s/n of the total
        assert prefix[b] * n >= total * s
        assert b == 0 or prefix[b - 1] * n < total * s
    # no shard exceeds its share by more than one sequence's work
    for s in range(n):
        assert prefix[bounds[s + 1]] - prefix[bounds[s]] <= total / n + max(work)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # forward: causal GQA, B=2, Hq=8, Hkv=2 (4 units), ragged length
        q, k, v = prefill_inputs(2, 8, 2, 70, 70, 16, seed=3)
        qv, kv, vv = fa.unit_views(q, k, v)
        first, count = fa.shard_units(2, 2, world, rank)
        o_s, l_s = oracle.attn_fwd(qv[first:first + count], kv[first:first + count],
                                   vv[first:first + count], True, 0.25)
        pieces = [None] * world
        dist.all_gather_object(pieces, (first, count, o_s, l_s))
        # decode: 6 sequences of different lengths, sharded by key count
        qd, kc, vc, sl = decode_inputs(6, 4, 2, 1, 90, 16, seed=4)
        bounds = fa.shard_sequences(sl, world)
        a, b = bounds[rank], bounds[rank + 1]
        od_s, ld_s = oracle.decode(qd[a:b], kc[a:b], vc[a:b], sl[a:b], 0.25)
        dec_pieces = [None] * world
        dist.all_gather_object(dec_pieces, (a, b, od_s, ld_s))
        if rank == 0:
            out["fwd"] = pieces
            out["dec"] = dec_pieces
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reassemble():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    q, k, v = prefill_inputs(2, 8, 2, 70, 70, 16, seed=3)
    o_ref, l_ref = oracle.attn_fwd(q, k, v, True, 0.25)
    o_ref, l_ref = o_ref.reshape(4, 4, 70, 16), l_ref.reshape(4, 4, 70)
    covered = 0
    for first, count, o_s, l_s in out["fwd"]:
        assert count > 0  # 4 units over 2 ranks
        assert np.array_equal(o_s, o_ref[first:first + count])
        assert np.array_equal(l_s, l_ref[first:first + count])
        covered += count
    assert covered == 4
    qd, kc, vc, sl = decode_inputs(6, 4, 2, 1, 90, 16, seed=4)
    od_ref, ld_ref = oracle.decode(qd, kc, vc, sl, 0.25)
    covered = 0
    for a, b, od_s, ld_s in out["dec"]:
        assert np.array_equal(od_s, od_ref[a:b]) and np.array_equal(ld_s, ld_ref[a:b])
        covered += b - a
    assert covered == 6


@pytest.mark.gpu
@pytest.mark.parametrize("host", [False, True])
def test_sharded_forward_equals_one_launch(host):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    q, k, v = prefill_inputs(2, 8, 2, 333, 333, 128, seed=21)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1 = torch.empty_like(qc)
    l1 = torch.empty((2, 8, 333), device="cuda")
    fa.fa_fwd(qc, kc, vc, o1, l1, True, 0.09)
    dev = torch.device("cuda", 0)
    src = (q.pin_memory(), k.pin_memory(), v.pin_memory()) if host else (qc, kc, vc)
    o2, l2 = fa.flash_attention_sharded(*src, causal=True, scale=0.09, devices=[dev, dev, dev])
    torch.cuda.synchronize()
    assert o2.is_cuda == (not host)
    assert torch.equal(o2.to(dev), o1) and torch.equal(l2.to(dev), l1)


@pytest.mark.gpu
def test_sharded_decode_equals_one_device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    q, kc, vc, sl = decode_inputs(6, 8, 2, 100, 2000, 128, seed=22, device="cuda")
    o1, l1 = fa.decode_attention(q, kc, vc, sl, num_splits=4)
    dev = torch.device("cuda", 0)
    o2, l2 = fa.decode_attention_sharded(q, kc, vc, sl, devices=[dev, dev], num_splits=4)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o_ref, l_ref = oracle.decode(q, kc, vc, sl, 1.0 / math.sqrt(128))
    assert float(np.abs(o2.float().cpu().numpy() - o_ref).max()) <= 2e-2
