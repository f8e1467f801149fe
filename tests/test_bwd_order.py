"""The backward's CTA order, checked on the host through fa_debug_bwd_tiles.

fa_bwd launches one CTA per (batch, kv head, key tile) for dK/dV and one per
(batch, query head, query tile) for dQ, in an order chosen per problem
(interleaved by head group, or by role).  Whatever the order, every unit must
be launched exactly once, and within one head the tiles must go out heaviest
first (under a causal mask key tile 0 and the last query tile see the most
work).  No GPU is needed: the order is computed by the same host and
host/device code the launch uses.
"""
import ctypes
from collections import Counter

import numpy as np
import pytest

from io_aware_exact_flashattention_b200 import fa


def bwd_tiles(B, Hq, Hkv, Sq, Skv, d, causal, sms):
    lib = fa.lib()
    n = ctypes.c_longlong(0)
    inter = ctypes.c_int(0)
    assert lib.fa_debug_bwd_tiles(B, Hq, Hkv, Sq, Skv, d, int(causal), sms, None, 0,
                                  ctypes.byref(n), ctypes.byref(inter)) == 0
    tiles = np.zeros((n.value, 4), dtype=np.int32)
    assert lib.fa_debug_bwd_tiles(B, Hq, Hkv, Sq, Skv, d, int(causal), sms,
                                  tiles.ctypes.data_as(ctypes.c_void_p), n.value,
                                  ctypes.byref(n), ctypes.byref(inter)) == 0
    return tiles, inter.value


SHAPES = [
    # B, Hq, Hkv, Sq, Skv, d, causal, sms
    (4, 16, 16, 2048, 2048, 128, True, 148),   # causal MHA S2048 (interleaved)
    (2, 32, 8, 8192, 8192, 128, True, 148),    # causal GQA S8192
    (1, 32, 8, 4096, 4096, 128, True, 148),    # long GQA dK/dV CTAs (by role)
    (1, 32, 8, 32768, 32768, 128, True, 148),  # causal GQA S32768
    (3, 6, 2, 700, 300, 64, True, 148),        # Sq > Skv, ragged tiles
    (2, 4, 1, 150, 400, 128, True, 148),       # Sq < Skv
    (2, 4, 2, 1000, 1000, 64, False, 148),     # non-causal
    (5, 8, 4, 513, 513, 128, True, 7),         # few SMs: many small groups
    (1, 2, 2, 128, 128, 64, True, 1),          # one SM, one tile
    (2, 4, 4, 256, 0, 128, True, 148),         # no keys: dQ CTAs only
]


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Skv,d,causal,sms", SHAPES)
def test_every_unit_once_heavy_first(B, Hq, Hkv, Sq, Skv, d, causal, sms):
    tiles, _ = bwd_tiles(B, Hq, Hkv, Sq, Skv, d, causal, sms)
    nkv = (Skv + 127) // 128
    nq = (Sq + 127) // 128
    assert len(tiles) == B * Hkv * nkv + B * Hq * nq
    want = Counter()
    for b in range(B):
        for g in range(Hkv):
            for j in range(nkv):
                want[(1, b, g, j)] += 1
        for h in range(Hq):
            for i in range(nq):
                want[(0, b, h, i)] += 1
    got = Counter(tuple(int(x) for x in row) for row in tiles)
    assert got == want
    # per head, in launch order: key tiles ascending, query tiles descending
    seen = {}
    for kv, b, hg, t in tiles:
        key = (int(kv), int(b), int(hg))
        if key in seen:
            prev = seen[key]
            assert (t > prev) if kv == 1 else (t < prev), (key, prev, t)
        seen[key] = int(t)


def test_order_modes_of_the_gpu_test_shapes():
    # the interleaved order on the headline backward shape, the by-role order on
    # the long-sequence GQA shape that tests/test_backward_gpu.py runs for it
    assert bwd_tiles(4, 16, 16, 2048, 2048, 128, True, 148)[1] == 1
    assert bwd_tiles(1, 32, 8, 4096, 4096, 128, True, 148)[1] == 0


def test_interleaved_groups_put_a_heads_dq_ctas_after_its_dkdv_ctas():
    tiles, inter = bwd_tiles(4, 16, 16, 2048, 2048, 128, True, 148)
    assert inter == 1
    last_kv = {}
    first_q = {}
    for pos, (kv, b, hg, t) in enumerate(tiles):
        if kv == 1:
            last_kv[(int(b), int(hg))] = pos
        else:
            first_q.setdefault((int(b), int(hg)), pos)  # MHA: query head = kv head
    for key, pos in last_kv.items():
        assert first_q[key] > pos


def test_argument_errors():
    lib = fa.lib()
    n = ctypes.c_longlong(0)
    inter = ctypes.c_int(0)
    bad = [
        (0, 4, 4, 128, 128, 128, 1, 148),   # B < 1
        (1, 6, 4, 128, 128, 128, 1, 148),   # Hq % Hkv != 0
        (1, 4, 4, 0, 128, 128, 1, 148),     # Sq < 1
        (1, 4, 4, 128, 128, 128, 1, 0),     # sms < 1
    ]
    for args in bad:
        assert lib.fa_debug_bwd_tiles(*args, None, 0, ctypes.byref(n), ctypes.byref(inter)) == 1
    assert lib.fa_debug_bwd_tiles(1, 4, 4, 128, 128, 96, 1, 148, None, 0, ctypes.byref(n),
                                  ctypes.byref(inter)) == 2
    # too small a buffer
    buf = np.zeros((1, 4), dtype=np.int32)
    assert lib.fa_debug_bwd_tiles(1, 4, 4, 512, 512, 128, 1, 148,
                                  buf.ctypes.data_as(ctypes.c_void_p), 1, ctypes.byref(n),
                                  ctypes.byref(inter)) == 1
