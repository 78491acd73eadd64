"""The product path has no CPU fallback and never reaches the oracle.

Every compute call of the binding refuses tensors that are not on a CUDA
device, before anything is computed; with the shared library missing, the
calls that need it raise and name the build command; the package's sources
neither import nor read anything under oracle/.  All of this runs without a
GPU.
"""
import os
import re

import pytest
import torch

import context_exact_attention_ring_b200 as ra
from context_exact_attention_ring_b200 import ring as R

PKG = os.path.dirname(os.path.abspath(ra.__file__))


def _cpu(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


B, S, HQ, HKV, D, P = 1, 256, 4, 2, 64, 2
q, k, v = _cpu(B, S, HQ, D), _cpu(B, S, HKV, D), _cpu(B, S, HKV, D)
out, lse = _cpu(B, S, HQ, D), _cpu(B, HQ, S, dtype=torch.float32)
dq1, dk1, dv1 = _cpu(B, 1, HQ, D), _cpu(B, S, HKV, D), _cpu(B, S, HKV, D)
sl = torch.full((B,), S, dtype=torch.int32)
m, l, O = _cpu(B, HQ, S // P, dtype=torch.float32), _cpu(B, HQ, S // P, dtype=torch.float32), \
    _cpu(B, S // P, HQ, D, dtype=torch.float32)

CALLS = {
    "ring_attn_fwd": lambda: ra.ring_attn_fwd(q, k, v, P),
    "ring_attn_fwd_counted": lambda: ra.ring_attn_fwd_counted(q, k, v, P, counters=torch.zeros(2 + P, dtype=torch.int64)),
    "ring_attn_fwd_simt": lambda: ra.ring_attn_fwd_simt(q, k, v, P),
    "ring_attn_bwd": lambda: ra.ring_attn_bwd(q, k, v, out, lse, out, P),
    "ring_attn_bwd_simt": lambda: ra.ring_attn_bwd_simt(q, k, v, out, lse, out, P),
    "ring_attn_bwd_delta": lambda: ra.ring_attn_bwd_delta(out, out),
    "ring_attn_state_init": lambda: ra.ring_attn_state_init(m, l, O),
    "ring_attn_step": lambda: ra.ring_attn_step(q[:, :S // P], k[:, :S // P], v[:, :S // P], m, l, O, [0], [0],
                                                S // P),
    "ring_attn_state_finalize": lambda: ra.ring_attn_state_finalize(m, l, O),
    "ring_attn_decode_partial": lambda: ra.ring_attn_decode_partial(q[:, 0], k, v, sl, P),
    "ring_attn_decode_partial_noalloc": lambda: ra.ring_attn_decode_partial_noalloc(q[:, 0], k, v, sl, P),
    "ring_attn_merge": lambda: ra.ring_attn_merge(_cpu(B, HQ, P, D, dtype=torch.float32),
                                                  _cpu(B, HQ, P, dtype=torch.float32)),
    "ring_attn_decode": lambda: ra.ring_attn_decode(q[:, 0], k, v, sl, P),
    "ring_attn_decode_fused": lambda: ra.ring_attn_decode_fused(q[:, 0], k, v, P, seqlens=sl),
    "ring_attn_kv_append": lambda: ra.ring_attn_kv_append(k, v, dk1[:, :, :HKV], dk1[:, :, :HKV],
                                                          torch.zeros((B, P), dtype=torch.int32),
                                                          torch.zeros((B,), dtype=torch.int32), P, 16),
    "ring_attn_step_bwd": lambda: ra.ring_attn_step_bwd(q[:, :S // P], k[:, :S // P], v[:, :S // P],
                                                        out[:, :S // P], lse[:, :, :S // P], lse[:, :, :S // P],
                                                        dq1, dk1, dv1, [0], [0], S // P),
    "ring.ring_forward (default step)": lambda: R.ring_forward(q, k, v, ring=_OneRank()),
}


class _OneRank:
    rank, world = 0, 1

    def shift(self, send, recv):
        return []


@pytest.mark.parametrize("name", sorted(CALLS))
def test_compute_calls_refuse_host_tensors(name):
    with pytest.raises(ValueError, match="CUDA device"):
        CALLS[name]()


def test_missing_library_raises_and_names_the_build(monkeypatch, tmp_path):
    monkeypatch.setattr(ra, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(ra, "_lib", None)
    with pytest.raises(RuntimeError, match="missing: build it with"):
        ra.ring_attn_sched_stats(1024, 4, True, "zigzag")
    with pytest.raises(RuntimeError, match="missing"):
        ra.ring_attn_decode_workspace_bytes(1, 4, 2, 1024, 64, 2)
    with pytest.raises(RuntimeError, match="missing"):
        ra.lib()


def test_package_sources_never_reach_the_oracle():
    pat = re.compile(r"\boracle\b")
    hits = []
    for root, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp", ".c")):
                path = os.path.join(root, f)
                for n, line in enumerate(open(path, encoding="utf-8"), 1):
                    if pat.search(line) and ("import" in line or "oracle/" in line or "oracle." in line):
                        hits.append(f"{os.path.relpath(path, PKG)}:{n}: {line.strip()}")
    assert not hits, "\n".join(hits)


def test_bench_reaches_the_oracle_only_in_its_cpu_baseline():
    # bench.py may run the oracle only for the timed CPU baseline (its cpu_baseline leg and the
    # reference arm, which calls it); every import of oracle must sit inside that function
    import ast
    root = os.path.dirname(PKG)
    tree = ast.parse(open(os.path.join(root, "bench.py"), encoding="utf-8").read())
    owners = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            name = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else fn
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                owners.append(fn)
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                owners.append(fn)
            visit(child, name)

    visit(tree, None)
    assert owners and set(owners) == {"cpu_baseline"}, owners
