"""The Helix decode exchange (context_exact_attention_ring_b200/ring.py,
helix_decode) on CPU ranks: world sizes 2 to 4 as gloo processes.  Rank r
holds shard r of every sequence's KV cache (some shards empty, some ragged),
computes the partial of every query head over it with a numpy stand-in for the
decode kernel, and the ranks exchange the partials with one all-gather; each
rank merges them (the oracle's merge formula stands in for the merge kernel).
Every rank must end with attention over all valid keys, checked against the
fp64 oracle.  A one-rank run on the GPU drives the real kernels."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from context_exact_attention_ring_b200 import ring as R

B, HQ, HKV, D, C = 3, 4, 2, 16, 24          # C rows per shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(world, seed=41):
    rng = np.random.default_rng(seed)
    f = lambda *shape: rng.standard_normal(shape).astype(np.float32)   # the oracle reads float32 values
    q = f(B, HQ, D)
    k = f(B, world * C, HKV, D)
    v = f(B, world * C, HKV, D)
    lens = np.array([world * C, C + 5, 7])[:B]            # full, ragged into shard 1, inside shard 0
    return q, k, v, lens


def fake_partial(q, k, v, lens, scale):
    """Attention of each query head over the shard's valid rows (numpy, float64):
    normalised O and lse; an empty shard gives O = 0, lse = -inf."""
    qn, kn, vn = q.double().numpy(), k.double().numpy(), v.double().numpy()
    G = qn.shape[1] // kn.shape[2]
    O = np.zeros((qn.shape[0], qn.shape[1], 1, qn.shape[2]))
    L = np.full((qn.shape[0], qn.shape[1], 1), -np.inf)
    for b in range(qn.shape[0]):
        n = int(lens[b])
        if n == 0:
            continue
        kh = np.repeat(kn[b, :n], G, axis=1)
        vh = np.repeat(vn[b, :n], G, axis=1)
        s = np.einsum("hd,nhd->hn", qn[b], kh) * scale
        m = s.max(-1)
        p = np.exp(s - m[:, None])
        z = p.sum(-1)
        O[b, :, 0] = np.einsum("hn,nhd->hd", p, vh) / z[:, None]
        L[b, :, 0] = m + np.log(z)
    return torch.from_numpy(O), torch.from_numpy(L)


def fake_merge(parts, lses):
    from oracle import merge as omerge
    o, l = omerge.merge(parts.numpy(), lses.numpy())
    return torch.from_numpy(o), torch.from_numpy(l)


def _rank(rank, world, port, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, lens = _inputs(world)
        sl = slice(rank * C, (rank + 1) * C)
        shard_len = torch.from_numpy(np.clip(lens - rank * C, 0, C).astype(np.int32))
        out, lse = R.helix_decode(torch.from_numpy(q), torch.from_numpy(np.ascontiguousarray(k[:, sl])),
                                  torch.from_numpy(np.ascontiguousarray(v[:, sl])), shard_len, scale=0.3,
                                  partial=fake_partial, merge=fake_merge)
        q_out.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
def test_helix_exchange_on_cpu_ranks(world):
    import oracle
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = [qq.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    q, k, v, lens = _inputs(world)
    G = HQ // HKV
    for b in range(B):
        for g in range(HKV):
            rows = [(0, i, 0) for i in range(G)]
            ro, rl = oracle.attention_rows(q[b:b + 1, None, g * G:(g + 1) * G], k[b:b + 1, :, g:g + 1],
                                           v[b:b + 1, :, g:g + 1], rows, scale=0.3, causal=False,
                                           kv_len=np.array([lens[b]]))
            for rank, out, lse in res:
                np.testing.assert_allclose(out[b, g * G:(g + 1) * G], ro, atol=1e-12, rtol=0)
                np.testing.assert_allclose(lse[b, g * G:(g + 1) * G], rl, atol=1e-12, rtol=0)



def _rank_round_robin(rank, world, block, port, q_out):
    # every sequence's tokens dealt to the ranks block by block, as ring_attn_kv_append places
    # them ("NVIDIA unveils Helix Parallelism", KV cache growth; oracle.helix simulates it)
    from oracle import helix
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, lens = _inputs(world, seed=43)
        cap = k.shape[1]
        ks = np.zeros((B, cap, HKV, D), np.float32)
        vs = np.zeros_like(ks)
        shard_len = np.zeros(B, np.int32)
        for b in range(B):
            shards, _, _, dropped = helix.simulate_appends([[] for _ in range(world)], 0, list(range(lens[b])),
                                                           block, world, cap)
            assert dropped == 0
            mine = shards[rank]
            ks[b, :len(mine)] = k[b, mine]
            vs[b, :len(mine)] = v[b, mine]
            shard_len[b] = len(mine)
        out, lse = R.helix_decode(torch.from_numpy(q), torch.from_numpy(ks), torch.from_numpy(vs),
                                  torch.from_numpy(shard_len), scale=0.3, partial=fake_partial, merge=fake_merge)
        q_out.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,block", [(2, 4), (3, 1), (4, 8)])
def test_helix_exchange_over_round_robin_shards(world, block):
    # a single query attends to the union of the shards in any order: the exchange over
    # round-robin shards equals attention over every token of the sequence
    import oracle
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_round_robin, args=(r, world, block, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = [qq.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    q, k, v, lens = _inputs(world, seed=43)
    G = HQ // HKV
    for b in range(B):
        for g in range(HKV):
            rows = [(0, i, 0) for i in range(G)]
            ro, rl = oracle.attention_rows(q[b:b + 1, None, g * G:(g + 1) * G], k[b:b + 1, :, g:g + 1],
                                           v[b:b + 1, :, g:g + 1], rows, scale=0.3, causal=False,
                                           kv_len=np.array([lens[b]]))
            for rank, out, lse in res:
                np.testing.assert_allclose(out[b, g * G:(g + 1) * G], ro, atol=1e-12, rtol=0)
                np.testing.assert_allclose(lse[b, g * G:(g + 1) * G], rl, atol=1e-12, rtol=0)

def _gpu_rank(port, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        import workloads as W
        cfg = W.Decode("helix1", 3, 16, 4, 128, 8192, 1, 51, fixed_lens=(8192, 3000, 1))
        q, k, v, sl = W.decode_inputs(cfg, "cuda")
        out, lse = R.helix_decode(q, k, v, sl, scale=cfg.scale)
        torch.cuda.synchronize()
        f = lambda t: t.float().cpu().numpy()
        q_out.put([f(q), f(k), f(v), sl.cpu().numpy(), f(out), f(lse)])
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_helix_exchange_one_gpu_rank_runs_the_kernels():
    # one NCCL rank: the decode kernel, the all-gather and the merge kernel against the fp64 oracle
    import oracle
    from tests.helpers import margin, need_cuda
    need_cuda()
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    p = ctx.Process(target=_gpu_rank, args=(_free_port(), qq))
    p.start()
    q, k, v, lens, out, lse = qq.get(timeout=300)
    p.join(60)
    assert p.exitcode == 0
    Bq, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    for b in range(Bq):
        for g in range(Hkv):
            rows = [(0, i, 0) for i in range(G)]
            ro, rl = oracle.attention_rows(q[b:b + 1, None, g * G:(g + 1) * G], k[b:b + 1, :, g:g + 1],
                                           v[b:b + 1, :, g:g + 1], rows, scale=1.0 / np.sqrt(D), causal=False,
                                           kv_len=np.array([lens[b]]))
            margin("out", np.max(np.abs(out[b, g * G:(g + 1) * G] - ro)), 2e-2)
            margin("lse", np.max(np.abs(lse[b, g * G:(g + 1) * G] - rl)), 1e-3)


def _rank_fails(rank, world, port, fail_rank, q_out):
    # a rank whose partial raises before the exchange; the others wait in the all-gather, and must
    # end with an error (its connection closes, or the process group's 5 s timeout runs out)
    import time
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    q, k, v, lens = _inputs(world)
    sl = slice(rank * C, (rank + 1) * C)
    shard_len = torch.from_numpy(np.clip(lens - rank * C, 0, C).astype(np.int32))

    def partial(*a):
        if rank == fail_rank:
            raise RuntimeError("planted failure in the partial")
        return fake_partial(*a)

    t0 = time.monotonic()
    try:
        R.helix_decode(torch.from_numpy(q), torch.from_numpy(np.ascontiguousarray(k[:, sl])),
                       torch.from_numpy(np.ascontiguousarray(v[:, sl])), shard_len, scale=0.3,
                       partial=partial, merge=fake_merge)
        q_out.put((rank, None, time.monotonic() - t0))
    except Exception as e:                                    # noqa: BLE001 -- any error ends the rank
        q_out.put((rank, f"{type(e).__name__}: {e}"[:200], time.monotonic() - t0))
    # no destroy_process_group: a peer is gone, and the process exits here


@pytest.mark.parametrize("world,fail_rank", [(2, 1), (3, 0)])
def test_a_rank_failing_before_the_exchange_ends_every_rank_with_an_error(world, fail_rank):
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_fails, args=(r, world, port, fail_rank, qq)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted(qq.get(timeout=90) for _ in range(world))
    finally:
        for p in procs:
            p.join(30)
            if p.is_alive():
                p.kill()                      # this test's own child, by its handle
                p.join(10)
    for rank, err, secs in res:
        # nobody can merge without every shard's partial
        assert err is not None, f"rank {rank} merged without rank {fail_rank}'s partial"
        if rank == fail_rank:
            assert "planted failure" in err
        assert secs < 60, (rank, secs)
