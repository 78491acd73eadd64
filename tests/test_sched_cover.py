"""The attention kernels' schedulers (csrc/ring_sched.h, csrc/bwd_sched.h),
walked on the host.

tests/sched_cover.cpp includes the scheduler headers the kernels use, builds
with g++ and walks every work item and step as the kernels do: the forward
tensor-core kernel, and both launches of the tensor-core backward (K/V-major
for dK and dV, Q-major for dQ).  For every split, rank count, chunk count,
ragged chunk length, GQA grouping, tile shape and mask, it checks the
following:
- each pair the causal rule allows is computed exactly once, and no other
  pair is;
- each output row has exactly one owner, so no two CTAs write the same row;
- every index stays inside its buffer;
- the step count the MMA warp expects equals the step count the producer
  walks.
This stands in on the CPU for the bounds and race checks a sanitizer would
make on the GPU.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
LAYOUT = {"contiguous": 0, "zigzag": 1, "striped": 2}


@pytest.fixture(scope="module")
def walker(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("sched") / "libsched_cover.so")
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-Wall", "-Werror", "-shared", "-fPIC", "-o", so,
                           os.path.join(HERE, "sched_cover.cpp")])
    lib = ctypes.CDLL(so)
    i, p = ctypes.c_int, ctypes.c_void_p
    lib.sched_cover_ring.argtypes = [i] * 11 + [p, ctypes.c_char_p]
    lib.sched_cover_step.argtypes = [i] * 5 + [p, i, p, i, i, i, i, i, p, ctypes.c_char_p]
    return lib


FORWARD, BACKWARD_KV, BACKWARD_Q, FORWARD_PAIR = 0, 1, 2, 3


def _ring(lib, B, Hq, Hkv, S, P, layout, cpr, causal, which=FORWARD, BM=128, BN=128):
    stats = np.zeros(3, np.int64)
    msg = ctypes.create_string_buffer(256)
    rc = lib.sched_cover_ring(B, Hq, Hkv, S, P, LAYOUT[layout], cpr, int(causal), which, BM, BN, stats.ctypes.data,
                              msg)
    assert rc == 0, (rc, msg.value.decode())
    return stats


CASES = []
for layout, cprs in (("contiguous", (1, 2, 3)), ("zigzag", (2, 3, 4, 8)), ("striped", (1,))):
    for cpr in cprs:
        for P in (1, 2, 3, 5, 8):
            for C in (64, 100, 257):             # one tile, ragged, several tiles with a ragged tail
                if P * cpr * C > 2100:
                    continue
                CASES.append((layout, cpr, P, C))


@pytest.mark.parametrize("which", [FORWARD, BACKWARD_KV, BACKWARD_Q, FORWARD_PAIR])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("layout,cpr,P,C", CASES)
def test_ring_mode_covers_each_allowed_pair_once(walker, layout, cpr, P, C, causal, which):
    S = P * cpr * C
    # even group: head pairs; odd group: two row tiles per item; the CTA-pair kernel also takes
    # four heads (group 4), or two heads at two row tiles (group 2), or four row tiles
    groups = ((2, 1), (3, 3), (4, 1), (8, 2)) if which == FORWARD_PAIR else ((2, 1), (3, 3))
    for Hq, Hkv in groups:
        stats = _ring(walker, 1, Hq, Hkv, S, P, layout, cpr, causal, which)
        allowed = S * (S + 1) // 2 if causal else S * S
        assert stats[2] == Hq * allowed


@pytest.mark.parametrize("BM,BN", [(128, 128), (128, 64), (64, 128)])
def test_tile_shapes_batches_and_gqa(walker, BM, BN):
    for (Hq, Hkv) in ((8, 2), (6, 3), (5, 1), (4, 4), (16, 2), (12, 2)):
        for which in (FORWARD, FORWARD_PAIR):
            _ring(walker, 2, Hq, Hkv, 4 * 2 * 200, 4, "zigzag", 2, True, which, BM, BN)
            _ring(walker, 2, Hq, Hkv, 3 * 130, 3, "striped", 1, True, which, BM, BN)


def test_backward_batches_and_gqa(walker):
    for which in (BACKWARD_KV, BACKWARD_Q):
        for (Hq, Hkv) in ((8, 2), (6, 3), (5, 1)):
            _ring(walker, 2, Hq, Hkv, 4 * 2 * 200, 4, "zigzag", 2, True, which)
            _ring(walker, 2, Hq, Hkv, 3 * 130, 3, "striped", 1, True, which)


@pytest.mark.parametrize("snake", [True, False])
def test_backward_deals_every_item_to_one_cta_turn(walker, snake):
    walker.sched_cover_turns.argtypes = [ctypes.c_int] * 3 + [ctypes.c_char_p]
    msg = ctypes.create_string_buffer(256)
    for grid in (1, 2, 3, 148):
        for items in (0, 1, grid - 1, grid, grid + 1, 2 * grid, 2 * grid + 5, 7 * grid + 3, 8192):
            if items < 0:
                continue
            rc = walker.sched_cover_turns(items, grid, int(snake), msg)
            assert rc == 0, (grid, items, rc, msg.value.decode())


def test_alternating_waves_keep_the_ctas_in_step(walker):
    # Items ordered longest first with work falling linearly along the order (the kernels'
    # orders): dealt in alternating wave order, the work a CTA has done after every second wave
    # differs from any other CTA's by at most one wave's spread of item lengths; dealt in the
    # same order every wave, the spread grows with every wave.
    walker.sched_turn_item.argtypes = [ctypes.c_int] * 5
    grid, items = 148, 148 * 40
    work = lambda L: 10_000 - L   # falls by one unit per item
    spread = {}
    for snake in (True, False):
        done = np.zeros(grid)
        worst = 0.0
        for w in range(items // grid):
            for c in range(grid):
                L = walker.sched_turn_item(w, c, grid, items, int(snake))
                done[c] += work(L)
            if w % 2 == 1:
                worst = max(worst, done.max() - done.min())
        spread[snake] = worst
    assert spread[True] <= grid - 1                    # one wave's spread at most
    assert spread[False] >= 20 * (grid - 1)            # 40 waves of the same spread, added up


def _step(lib, C, qid, kid, stripes, causal, Hq=2, Hkv=1, which=FORWARD):
    stats = np.zeros(3, np.int64)
    msg = ctypes.create_string_buffer(256)
    q = (ctypes.c_int * len(qid))(*qid)
    k = (ctypes.c_int * len(kid))(*kid)
    rc = lib.sched_cover_step(1, Hq, Hkv, C, len(qid), ctypes.cast(q, ctypes.c_void_p), len(kid),
                              ctypes.cast(k, ctypes.c_void_p), stripes, int(causal), which, 128, 128,
                              stats.ctypes.data, msg)
    assert rc == 0, (rc, msg.value.decode())
    return stats


@pytest.mark.parametrize("which", [FORWARD, BACKWARD_KV, BACKWARD_Q, FORWARD_PAIR])
@pytest.mark.parametrize("causal", [True, False])
def test_step_mode_covers_each_allowed_pair_of_the_held_block_once(walker, causal, which):
    # every (query shard, held block) pair of a zig-zag ring with P = 4 (8 chunks), chunk length 200,
    # and shards given in either chunk order
    P = 4
    own = [[r, 2 * P - 1 - r] for r in range(P)]
    for r in range(P):
        for s in range(P):
            for q_ids in (own[r], own[r][::-1]):
                st = _step(walker, 200, q_ids, own[s], 0, causal, which=which)
                qt = [c * 200 + x for c in q_ids for x in range(200)]
                kt = [c * 200 + y for c in own[s] for y in range(200)]
                expect = sum(1 for a in qt for b in kt if b <= a) if causal else len(qt) * len(kt)
                assert st[2] == 2 * expect


@pytest.mark.parametrize("which", [FORWARD, BACKWARD_KV, BACKWARD_Q, FORWARD_PAIR])
def test_step_mode_stripes(walker, which):
    P, C = 5, 150
    for r in range(P):
        for s in range(P):
            st = _step(walker, C, [r], [s], P, True, Hq=3, Hkv=3, which=which)
            expect = sum(1 for x in range(C) for y in range(C) if y * P + s <= x * P + r)
            assert st[2] == 3 * expect

