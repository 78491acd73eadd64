"""Host-side tests of the C ABI (no GPU needed): the library loads and exports
every function include/ring_attn.h declares, argument checks return their
documented codes without touching a device, and the scheduler's host view
(ring_attn_sched_stats) equals the oracle's enumeration exactly."""
import ctypes
import os
import re

import pytest

import context_exact_attention_ring_b200 as ra
from oracle import schedule as sch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ring_attn.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from context_exact_attention_ring_b200 import build
    build.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(ring_attn_[a-z0-9_]+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_three_core_calls():
    names = declared_functions()
    for n in ("ring_attn_fwd", "ring_attn_step", "ring_attn_merge"):
        assert n in names


def test_every_declared_symbol_is_exported():
    L = ra.lib()
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(ra.EXPORTED) <= set(names)


def test_version_and_arch():
    assert ra.lib().ring_attn_version() >= 1
    assert ra.lib().ring_attn_built_arch() == 100


def test_strerror():
    for s in (0, -1, -2, -3, -4):
        assert ra.strerror(s)
    assert ra.strerror(-4) != ra.strerror(-1)


FAKE = 0x10000  # aligned, non-null; never dereferenced: every case below fails before any launch


def fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, S=256, D=64, P=4, causal=1, layout=0,
             scale=0.125, dtype=1)
    a.update(kw)
    return ra.lib().ring_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["S"],
                                  a["D"], a["P"], a["causal"], a["layout"], a["scale"], a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), ra.RING_EINVAL), (dict(lse=None), ra.RING_EINVAL), (dict(k=FAKE + 4), ra.RING_EINVAL),
    (dict(B=0), ra.RING_EINVAL), (dict(Hq=3), ra.RING_EINVAL), (dict(S=250), ra.RING_EINVAL),
    (dict(layout=1, S=260), ra.RING_EINVAL), (dict(layout=7), ra.RING_EINVAL), (dict(dtype=5), ra.RING_EINVAL),
    (dict(scale=0.0), ra.RING_EINVAL), (dict(scale=float("nan")), ra.RING_EINVAL), (dict(P=0), ra.RING_EINVAL),
    (dict(D=96), ra.RING_EUNSUPPORTED), (dict(D=256), ra.RING_EUNSUPPORTED),
    # split codes: zig-zag needs 2..8 chunks per rank, striped exactly one, S divisible by the chunks
    (dict(layout=ra.ring_split("zigzag", 1)), ra.RING_EINVAL), (dict(layout=ra.ring_split("zigzag", 9)), ra.RING_EINVAL),
    (dict(layout=ra.ring_split("striped", 2)), ra.RING_EINVAL), (dict(layout=ra.ring_split("contiguous", 9)), ra.RING_EINVAL),
    (dict(layout=ra.ring_split("zigzag", 3), S=260), ra.RING_EINVAL), (dict(layout=2, S=258), ra.RING_EINVAL),
    (dict(layout=1 << 16), ra.RING_EINVAL), (dict(layout=-1), ra.RING_EINVAL),
    (dict(layout=ra.ring_split("zigzag", 4), D=96), ra.RING_EUNSUPPORTED),
    (dict(layout=ra.ring_split("striped", 1), D=96), ra.RING_EUNSUPPORTED),
])
def test_fwd_argument_checks(kw, code):
    assert fwd(**kw) == code


def test_step_argument_checks():
    L = ra.lib()
    ids = ra.ChunkIds()
    ids.n_q, ids.n_kv, ids.chunk_len, ids.causal = 1, 1, 64, 1
    ids.q[0], ids.kv[0] = 0, 0
    args = lambda i, D=64: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(i), 1, 2, 2, D, 0.125, 1, None)
    assert L.ring_attn_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 2, 2, 64, 0.125, 1, None) == ra.RING_EINVAL
    bad = ra.ChunkIds(); ctypes.pointer(bad)[0] = ids; bad.kv[0] = -1
    assert L.ring_attn_step(*args(bad)) == ra.RING_EINVAL
    bad = ra.ChunkIds(); ctypes.pointer(bad)[0] = ids; bad.chunk_len = 0
    assert L.ring_attn_step(*args(bad)) == ra.RING_EINVAL
    bad = ra.ChunkIds(); ctypes.pointer(bad)[0] = ids; bad.n_q = ra.RING_MAX_CHUNKS_PER_RANK + 1
    assert L.ring_attn_step(*args(bad)) == ra.RING_EINVAL
    bad = ra.ChunkIds(); ctypes.pointer(bad)[0] = ids; bad.stripes = -1
    assert L.ring_attn_step(*args(bad)) == ra.RING_EINVAL
    bad = ra.ChunkIds(); ctypes.pointer(bad)[0] = ids; bad.stripes = 4; bad.kv[0] = 4   # rank outside the stripes
    assert L.ring_attn_step(*args(bad)) == ra.RING_EINVAL
    bad = ra.ChunkIds(); ctypes.pointer(bad)[0] = ids; bad.stripes = 4; bad.n_q = 2      # one stripe per shard
    assert L.ring_attn_step(*args(bad)) == ra.RING_EINVAL
    assert L.ring_attn_step(*args(ids, D=80)) == ra.RING_EUNSUPPORTED
    ok = ra.ChunkIds(); ctypes.pointer(ok)[0] = ids; ok.n_q = ok.n_kv = 8; ok.chunk_len = 8
    assert L.ring_attn_step(*args(ok, D=80)) == ra.RING_EUNSUPPORTED   # 8 chunks pass the id checks


def test_chunk_ids_struct_matches_header():
    # n_q, q[8], n_kv, kv[8], chunk_len, causal, stripes: 21 int32
    text = open(HEADER).read()
    assert "#define RING_MAX_CHUNKS_PER_RANK 8" in text
    assert ctypes.sizeof(ra.ChunkIds) == 4 * (3 + 2 * ra.RING_MAX_CHUNKS_PER_RANK + 2)


def test_decode_and_merge_argument_checks():
    L = ra.lib()
    ws = ra.ring_attn_decode_workspace_bytes(8, 32, 8, 1 << 20, 128, 32)
    assert ws > 0
    assert ra.ring_attn_decode_workspace_bytes(8, 32, 8, 1000, 128, 32) == 0      # Smax % P
    base = dict(q=FAKE, k=FAKE, v=FAKE, sl=FAKE, part=FAKE, plse=FAKE, B=8, Hq=32, Hkv=8, Smax=1 << 20, D=128, P=32,
                scale=0.088, dtype=0, ws=FAKE * 16, wsb=ws)

    def dec(**kw):
        a = dict(base); a.update(kw)
        return L.ring_attn_decode_partial(a["q"], a["k"], a["v"], a["sl"], a["part"], a["plse"], a["B"], a["Hq"],
                                          a["Hkv"], a["Smax"], a["D"], a["P"], a["scale"], a["dtype"], a["ws"],
                                          a["wsb"], None)
    assert dec(sl=None) == ra.RING_EINVAL
    assert dec(Smax=1000) == ra.RING_EINVAL
    assert dec(wsb=ws - 1) == ra.RING_EINVAL
    assert dec(ws=FAKE + 16) == ra.RING_EINVAL          # workspace must be 256-byte aligned
    assert dec(D=96) == ra.RING_EUNSUPPORTED             # head dimensions 64 and 128 are built
    assert dec(dtype=1) == ra.RING_EUNSUPPORTED
    assert dec(Hq=24) == ra.RING_EUNSUPPORTED            # GQA group of 3 is not built (1, 2, 4, 8, 16 are)
    assert L.ring_attn_merge(FAKE, FAKE, None, None, 1, 1, 1, 128, 0, None) == ra.RING_EINVAL
    assert L.ring_attn_merge(FAKE, FAKE, FAKE, None, 1, 1, 1, 130, 0, None) == ra.RING_EUNSUPPORTED
    assert L.ring_attn_merge(FAKE, FAKE, FAKE, None, 1, 1, 0, 128, 0, None) == ra.RING_EINVAL


@pytest.mark.parametrize("S,P,layout,causal,tq,tk", [
    (256, 4, "contiguous", False, 64, 64), (8192, 8, "contiguous", True, 128, 128),
    (32768, 8, "zigzag", True, 128, 128), (131072, 16, "zigzag", True, 128, 128),
    (1536, 3, "zigzag", True, 128, 128), (1000, 4, "zigzag", True, 128, 128), (960, 5, "contiguous", True, 64, 128),
    (3072, 4, "zigzag3", True, 128, 128), (131072, 16, "zigzag4", True, 128, 128), (4000, 2, "zigzag8", True, 64, 128),
    (8192, 4, "contiguous2", True, 128, 128), (131072, 16, "striped", True, 128, 128), (4096, 8, "striped", True, 128, 64),
    (1000, 4, "striped", True, 128, 128), (2048, 4, "striped", False, 128, 128), (1200, 3, "zigzag5", False, 64, 64),
])
def test_sched_stats_equals_oracle_enumeration(S, P, layout, causal, tq, tk):
    per, full, partial, skipped = ra.ring_attn_sched_stats(S, P, causal, layout, tq, tk)
    o_full, o_partial, o_skipped, _ = sch.tile_classes(S, P, layout, causal, tq, tk)
    assert (full, partial, skipped) == (o_full, o_partial, o_skipped)
    assert per == sch.per_rank_pairs(P, layout, causal, S)


def test_sched_stats_zigzag_closed_form():
    for P in (2, 8, 16):
        per, *_ = ra.ring_attn_sched_stats(64 * 2 * P, P, True, "zigzag")
        assert per == [2 * P + 1] * P
        per, *_ = ra.ring_attn_sched_stats(64 * P, P, True, "contiguous")
        assert per == [r + 1 for r in range(P)]


def test_header_builds_as_c_and_cxx_and_links_every_symbol(tmp_path):
    # a C99 program that includes the header, takes the address of every declared function (so
    # the linker must resolve each against the library) and calls the host-only entry points
    import subprocess
    names = declared_functions()
    lib_dir = os.path.dirname(ra.LIB_PATH)
    src = tmp_path / "use_abi.c"
    src.write_text(
        "#include <stdio.h>\n#include \"ring_attn.h\"\n"
        "typedef void (*fn_t)(void);\n"
        "int main(void) {\n"
        "  const fn_t fns[] = {" + ", ".join(f"(fn_t)&{n}" for n in names) + "};\n"
        "  size_t i, n = sizeof(fns) / sizeof(fns[0]);\n"
        "  int64_t per[4], f = 0, p = 0, s = 0;\n"
        "  for (i = 0; i < n; ++i) if (!fns[i]) return 2;\n"
        "  if (ring_attn_sched_stats(1024, 4, 1, RING_ZIGZAG, 128, 128, per, &f, &p, &s) != RING_OK) return 3;\n"
        "  printf(\"%d|%d|%s|%lld|%lld|%lld|%lld\\n\", ring_attn_version(), ring_attn_built_arch(),\n"
        "         ring_attn_strerror(RING_EINVAL), (long long)per[0], (long long)f, (long long)p, (long long)s);\n"
        "  return 0;\n}\n")
    exe = str(tmp_path / "use_abi")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                           os.path.join(ROOT, "include"), str(src), "-o", exe, "-L", lib_dir, "-lringattn_sm100a",
                           f"-Wl,-rpath,{lib_dir}"])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    ver, arch, err, per0, f, p, s = out.stdout.strip().split("|")
    assert int(arch) == 100 and int(ver) >= 1 and err == ra.strerror(ra.RING_EINVAL)
    # zig-zag, S = 1024, P = 4, 128-token tiles: 8 tiles per side, 2P+1 = 9 pairs per rank
    assert (int(per0), int(f), int(p), int(s)) == (9, 28, 8, 28)
    # the same header as C++ (its extern "C" block)
    cxx = tmp_path / "use_abi.cpp"
    cxx.write_text("#include \"ring_attn.h\"\nint main() { return ring_attn_version() > 0 ? 0 : 1; }\n")
    subprocess.check_call(["g++", "-std=c++11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                           os.path.join(ROOT, "include"), "-fsyntax-only", str(cxx)])


def test_backward_argument_checks():
    # every case fails a check before the first launch (the plan, then pointers, then the workspace)
    L = ra.lib()
    ws_need = L.ring_attn_bwd_workspace_bytes(1, 2, 256)
    assert ws_need == 2048 and L.ring_attn_bwd_workspace_bytes(0, 2, 256) == 0

    def bwd(fn=L.ring_attn_bwd, **kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, Hq=2, Hkv=2,
                 S=256, D=64, P=4, causal=1, layout=0, scale=0.125, dtype=0, ws=FAKE * 16, wsb=ws_need)
        a.update(kw)
        return fn(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], a["dq"], a["dk"], a["dv"], a["B"], a["Hq"],
                  a["Hkv"], a["S"], a["D"], a["P"], a["causal"], a["layout"], a["scale"], a["dtype"], a["ws"], a["wsb"],
                  None)
    for fn in (L.ring_attn_bwd, L.ring_attn_bwd_simt):
        assert bwd(fn, dout=None) == ra.RING_EINVAL
        assert bwd(fn, dq=FAKE + 8) == ra.RING_EINVAL
        assert bwd(fn, ws=None) == ra.RING_EINVAL
        assert bwd(fn, ws=FAKE + 16) == ra.RING_EINVAL          # 256-byte alignment
        assert bwd(fn, wsb=ws_need - 1) == ra.RING_EINVAL
        assert bwd(fn, S=250) == ra.RING_EINVAL
        assert bwd(fn, Hq=3) == ra.RING_EINVAL
        assert bwd(fn, D=96) == ra.RING_EUNSUPPORTED
    assert L.ring_attn_bwd_delta(None, FAKE, FAKE, 1, 2, 256, 64, 0, None) == ra.RING_EINVAL
    assert L.ring_attn_bwd_delta(FAKE, FAKE, FAKE, 0, 2, 256, 64, 0, None) == ra.RING_EINVAL
    assert L.ring_attn_bwd_delta(FAKE, FAKE, FAKE, 1, 2, 256, 64, 5, None) == ra.RING_EINVAL
    ids = ra.ChunkIds()
    ids.n_q, ids.n_kv, ids.chunk_len, ids.causal = 1, 1, 64, 1
    step = lambda i, dout=FAKE, D=64: L.ring_attn_step_bwd(FAKE, FAKE, FAKE, dout, FAKE, FAKE, FAKE, FAKE, FAKE, i, 1,
                                                          2, 2, D, 0.125, 0, None)
    assert step(None) == ra.RING_EINVAL
    assert step(ctypes.byref(ids), dout=FAKE + 4) == ra.RING_EINVAL
    assert step(ctypes.byref(ids), D=96) == ra.RING_EUNSUPPORTED


def test_fused_decode_and_append_argument_checks():
    L = ra.lib()
    ws = ra.ring_attn_decode_workspace_bytes(2, 8, 2, 4096, 128, 4)

    def fused(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, sl=FAKE, shard=None, part=FAKE, plse=FAKE, out=FAKE, olse=FAKE, B=2, Hq=8,
                 Hkv=2, Smax=4096, D=128, P=4, scale=0.088, dtype=0, ws=FAKE * 16, wsb=ws)
        a.update(kw)
        return L.ring_attn_decode_fused(a["q"], a["k"], a["v"], a["sl"], a["shard"], a["part"], a["plse"], a["out"],
                                        a["olse"], a["B"], a["Hq"], a["Hkv"], a["Smax"], a["D"], a["P"], a["scale"],
                                        a["dtype"], a["ws"], a["wsb"], None)
    assert fused(sl=None) == ra.RING_EINVAL                     # no source of lengths
    assert fused(shard=FAKE) == ra.RING_EINVAL                  # two sources of lengths
    assert fused(out=None) == ra.RING_EINVAL
    assert fused(olse=FAKE + 2) == ra.RING_EINVAL
    assert fused(wsb=ws - 1) == ra.RING_EINVAL
    assert fused(Hq=6) == ra.RING_EUNSUPPORTED                  # GQA group of 3

    def append(**kw):
        a = dict(kc=FAKE, vc=FAKE, kn=FAKE, vn=FAKE, sl=FAKE, na=FAKE, B=2, T=3, Hkv=2, Smax=4096, D=128, P=4, block=16,
                 dtype=0)
        a.update(kw)
        return L.ring_attn_kv_append(a["kc"], a["vc"], a["kn"], a["vn"], a["sl"], a["na"], a["B"], a["T"], a["Hkv"],
                                     a["Smax"], a["D"], a["P"], a["block"], a["dtype"], None)
    assert append(sl=None) == ra.RING_EINVAL
    assert append(kn=FAKE + 8) == ra.RING_EINVAL
    assert append(block=0) == ra.RING_EINVAL
    assert append(Smax=4095) == ra.RING_EINVAL                  # Smax % P
    assert append(T=0) == ra.RING_EINVAL
    assert append(dtype=5) == ra.RING_EINVAL
    assert append(Hkv=1, D=4) == ra.RING_EUNSUPPORTED           # a row of 8 bytes: rows move in 16-byte pieces


def test_sched_stats_random_sweep_equals_oracle_enumeration():
    # seeded random splits, rank counts, ragged chunk lengths and odd tile sizes
    import numpy as np
    rng = np.random.default_rng(77)
    layouts = ["contiguous", "contiguous2", "contiguous3", "zigzag", "zigzag3", "zigzag4", "zigzag6", "striped"]
    n = 0
    while n < 60:
        layout = layouts[rng.integers(len(layouts))]
        P = int(rng.integers(1, 7))
        k = sch.parse_layout(layout)[1]
        C = int(rng.integers(1, 300))
        S = P * k * C
        if S > 3000:
            continue
        tq, tk = int(rng.choice([16, 32, 48, 64, 100, 128])), int(rng.choice([16, 32, 64, 96, 128]))
        causal = bool(rng.integers(2))
        per, full, partial, skipped = ra.ring_attn_sched_stats(S, P, causal, layout, tq, tk)
        o_full, o_partial, o_skipped, _ = sch.tile_classes(S, P, layout, causal, tq, tk)
        assert (full, partial, skipped) == (o_full, o_partial, o_skipped), (S, P, layout, causal, tq, tk)
        assert per == sch.per_rank_pairs(P, layout, causal, S), (S, P, layout, causal)
        n += 1


def test_state_init_and_finalize_argument_checks():
    L = ra.lib()
    assert L.ring_attn_state_init(None, FAKE, FAKE, 1, 2, 64, 64, None) == ra.RING_EINVAL
    assert L.ring_attn_state_init(FAKE, FAKE + 4, FAKE, 1, 2, 64, 64, None) == ra.RING_EINVAL
    assert L.ring_attn_state_init(FAKE, FAKE, FAKE, 1, 2, 0, 64, None) == ra.RING_EINVAL
    assert L.ring_attn_state_init(FAKE, FAKE, FAKE, 1, 2, 64, 66, None) == ra.RING_EINVAL    # D % 4
    fin = lambda **kw: L.ring_attn_state_finalize(*[kw.get(n, FAKE) for n in ("m", "l", "O", "out", "lse")],
                                                  kw.get("B", 1), 2, 64, 64, kw.get("dtype", 0), None)
    assert fin(lse=None) == ra.RING_EINVAL
    assert fin(out=FAKE + 2) == ra.RING_EINVAL
    assert fin(B=0) == ra.RING_EINVAL
    assert fin(dtype=3) == ra.RING_EINVAL


def test_every_declared_function_documents_its_errors():
    # the comment above each declaration says what the call returns on failure (or that it cannot fail)
    text = open(HEADER).read()
    documented = {}
    for m in re.finditer(r"/\*(.*?)\*/\s*(?:#define[^\n]*\n)?([^;/]*?\b(ring_attn_[a-z0-9_]+)\s*\([^;]*;)", text, re.S):
        documented[m.group(3)] = bool(re.search(r"RING_E|[Ee]rrors|Returns|0 on bad|[Nn]ever fail", m.group(1)))
    assert set(declared_functions()) <= set(documented) | {"ring_attn_built_arch"}
    assert [n for n, ok in documented.items() if not ok] == []


def test_every_declared_function_cites_its_passage_or_says_it_has_none():
    text = open(HEADER).read()
    uncited = [m.group(3) for m in re.finditer(
        r"/\*(.*?)\*/\s*(?:#define[^\n]*\n)?([^;/]*?\b(ring_attn_[a-z0-9_]+)\s*\([^;]*;)", text, re.S)
        if not re.search(r"Lesson 8|Sequence parallelism|Helix|pages", m.group(1))]
    assert uncited == []


def test_binding_signatures_match_the_header():
    # the ctypes argument list of every bound function has the header's arity, with pointers where
    # the header has pointers, float where it has float and size_t where it has size_t
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    L = ra.lib()
    checked = 0
    for m in re.finditer(r"\b(ring_attn_[a-z0-9_]+)\s*\(([^;]*?)\)\s*;", text, flags=re.S):
        name, params = m.group(1), " ".join(m.group(2).split())
        fn = getattr(L, name)
        if fn.argtypes is None:
            continue
        params = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        assert len(params) == len(fn.argtypes), (name, params, fn.argtypes)
        for p, a in zip(params, fn.argtypes):
            if "*" in p:
                assert a in (ctypes.c_void_p,) or issubclass(a, ctypes._Pointer), (name, p, a)
            elif p.startswith("float "):
                assert a is ctypes.c_float, (name, p, a)
            elif p.startswith("size_t "):
                assert a is ctypes.c_size_t, (name, p, a)
            else:
                assert a is ctypes.c_int, (name, p, a)
        checked += 1
    assert checked >= 20
