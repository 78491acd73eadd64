"""Multi-GPU runs of bench.py are independent replicas (no collective on the
data path); only the timing is aggregated across ranks.  This checks that
aggregation with two gloo ranks on the CPU: the max over ranks and the
whole-job rate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [120.0, 150.0][rank]
        mx = bench.max_over_ranks(dist, local_ms, device="cpu")
        rate = bench.replica_throughput(1.0e12, 4, world, mx)
        q.put((rank, mx, rate))
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_and_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for _, mx, rate in res:
        assert mx == 150.0                                  # max over ranks
        assert rate == pytest.approx(1.0e12 * 4 * 2 / 0.150)  # all ranks' work / slowest rank's time


def test_single_process_is_identity():
    assert bench.max_over_ranks(None, 3.5) == 3.5
    assert bench.replica_throughput(2.0, 3, 1, 1000.0) == pytest.approx(6.0)


def test_cpu_baseline_small_sample():
    import workloads as W
    cfg = W.Prefill("tiny", "bf16", True, "zigzag", 1, 2, 1, 512, 64, 2, 3)
    r = bench.cpu_baseline(cfg, seconds=0.2)
    assert r["kind"] == "oracle" and r["cores"] >= 1 and r["value"] > 0 and r["unit"] == "TFLOP/s"



def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    # a copy of the kernel sources with traffic.json hashes matching them reports every kernel's
    # bytes; changing one byte of one kernel's source turns that kernel's traffic into None
    import hashlib
    import json
    import shutil
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for e in d.values():
        if not isinstance(e, dict):
            continue
        m = hashlib.sha256()
        for src in e["sources"]:
            dst = tmp_path / src
            dst.parent.mkdir(parents=True, exist_ok=True)
            shutil.copy(os.path.join(bench.ROOT, src), dst)
            m.update(dst.read_bytes())
        e["source_sha256"] = m.hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(d))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    cur = bench.load_traffic()
    assert cur["attn_tc_pair"] == d["attn_tc_pair"]["bytes"] and cur["decode"] == d["decode"]["bytes"]
    f = tmp_path / "context_exact_attention_ring_b200" / "csrc" / "decode.cu"
    f.write_text(f.read_text() + "\n")
    changed = bench.load_traffic()
    assert changed["decode"] is None and changed["attn_tc_pair"] == cur["attn_tc_pair"]


def test_profile_summaries_name_commands_the_bench_accepts():
    # every command a profile summary cites runs committed code: bench.py with options it
    # defines and profile cases it has
    import glob
    import re
    import shlex
    lines = []
    for f in glob.glob(os.path.join(bench.ROOT, "profiles", "*.md")):
        for line in open(f, encoding="utf-8"):
            if "python bench.py" in line:
                lines.append(line[line.index("python bench.py"):].strip())
    assert lines
    parser_src = open(os.path.join(bench.ROOT, "bench.py"), encoding="utf-8").read()
    options = set(re.findall(r'add_argument\("(--[a-z0-9-]+)"', parser_src))
    for cmd in lines:
        words = shlex.split(cmd)[2:]
        for i, w in enumerate(words):
            if w.startswith("--"):
                assert w in options, (cmd, w)
            if w == "--profile":
                assert words[i + 1] in bench.PROFILE_CASES, cmd
