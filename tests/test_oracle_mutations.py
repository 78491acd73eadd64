"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a scratch copy of oracle/: a dropped term, a
wrong sign, index or comparison, a transposed operand, the ring turning the
wrong way.  It then runs the pin tests that cover the mutated function in
that copy, and every planted mistake must make one of them fail.  A pin set
that lets a mistake through is too weak to vouch for the oracle.  Nothing here
touches the repository's own oracle files, and no GPU is involved.

The unmutated copy must pass the same pins.  That control shows that the
scratch tree is sound.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

ATTN = ["tests/test_oracle_attention.py"]
BWD = ["tests/test_oracle_backward.py"]
SCHED = ["tests/test_oracle_schedule.py"]
HELIX = ["tests/test_oracle_helix.py"]

# (name, file under oracle/, text to replace (must occur once), replacement, pin files)
MUTATIONS = [
    # attn_fp64.c, forward rows: the plain definition of attention ("Lesson 8: Context Parallelism",
    # section 1) with the causal rule of section 4
    ("causal rule drops the diagonal", "attn_fp64.c",
     "(!J->causal || kp <= qp)", "(!J->causal || kp < qp)", ATTN),
    ("GQA maps heads round-robin", "attn_fp64.c",
     "  const int g = h / G;\n  const int D = J->D;", "  const int g = h % J->Hkv;\n  const int D = J->D;", ATTN),
    ("scale dropped from the scores", "attn_fp64.c",
     "    s[j] = J->scale * acc;\n    if (s[j] > m) m = s[j];\n    any = 1;",
     "    s[j] = acc;\n    if (s[j] > m) m = s[j];\n    any = 1;", ATTN),
    ("row max dropped from lse", "attn_fp64.c",
     "J->lse[r] = m + log(Z);", "J->lse[r] = log(Z);", ATTN),
    ("output not normalised", "attn_fp64.c",
     "  for (int d = 0; d < D; ++d) o[d] /= Z;\n", "", ATTN),
    ("values read from K", "attn_fp64.c",
     "const float *vj = J->v + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;\n    const double w",
     "const float *vj = J->k + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;\n    const double w", ATTN),
    ("key length off by one", "attn_fp64.c",
     "(j < nkeys)", "(j <= nkeys && j < J->Skv)", ATTN),
    ("exponent sign flipped", "attn_fp64.c",
     "s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);", ATTN),
    ("query positions ignored", "attn_fp64.c",
     "const int64_t qp = J->qpos ? J->qpos[i] : i;\n  const int64_t nkeys",
     "const int64_t qp = i;\n  const int64_t nkeys", ATTN),
    ("key positions ignored", "attn_fp64.c",
     "const int64_t kp = J->kpos ? J->kpos[j] : j;\n    const int allowed",
     "const int64_t kp = j;\n    const int allowed", ATTN),
    # attn_fp64.c, backward: the calculus of the same definition
    ("softmax derivative drops delta", "attn_fp64.c",
     "const double ds = p * (dp[j] - delta);", "const double ds = p * dp[j];", BWD),
    ("dV weighted by dS", "attn_fp64.c",
     "dvj[d] += p * (double)oi[d];", "dvj[d] += ds * (double)oi[d];", BWD),
    ("dK missing the scale", "attn_fp64.c",
     "dkj[d] += J->scale * ds * (double)qi[d];", "dkj[d] += ds * (double)qi[d];", BWD),
    ("dQ sign flipped", "attn_fp64.c",
     "            dqi[d] += J->scale * ds * (double)kj[d];\n            dkj",
     "            dqi[d] -= J->scale * ds * (double)kj[d];\n            dkj", BWD),
    ("backward causal rule drops the diagonal", "attn_fp64.c",
     "if (J->causal && kp > qp)", "if (J->causal && kp >= qp)", BWD),
    ("backward ignores query positions", "attn_fp64.c",
     "const int64_t qp = J->qpos ? J->qpos[i] : i;\n        double m",
     "const int64_t qp = i;\n        double m", BWD),
    ("backward ignores key positions", "attn_fp64.c",
     "const int64_t kp = J->kpos ? J->kpos[j] : j;\n          if (J->causal",
     "const int64_t kp = j;\n          if (J->causal", BWD),
    ("sampled dQ rows drop the diagonal key", "attn_fp64.c",
     "const int nj = J->causal ? i + 1 : J->S;", "const int nj = J->causal ? i : J->S;", BWD),
    ("sampled dQ rows drop delta", "attn_fp64.c",
     "    for (int j = 0; j < nj; ++j) delta += exp(s[j] - lse) * dp[j];\n", "", BWD),
    # brute.py: the second, independent definition
    ("brute GQA maps heads round-robin", "brute.py",
     "kh = np.repeat(k, G, axis=2)", "kh = np.tile(k, (1, 1, G, 1))", ATTN),
    ("brute masks the diagonal", "brute.py",
     "(kp[None, :] <= qp[:, None])", "(kp[None, :] < qp[:, None])", ATTN),
    # merge.py: combining partial results ("NVIDIA unveils Helix Parallelism", KV parallelism)
    ("merge lse drops the max", "merge.py",
     "m[..., 0] + np.log(z_safe[..., 0])", "np.log(z_safe[..., 0])", ATTN),
    ("merge not normalised", "merge.py",
     "out = (w[..., None] * O).sum(axis=-2) / z_safe", "out = (w[..., None] * O).sum(axis=-2)", ATTN),
    # streaming.py: the online-softmax recurrence ("Lesson 8", section 3)
    ("recurrence forgets to rescale O", "streaming.py",
     "O * (alpha * l / l_div)[:, None]", "O * (l / l_div)[:, None]", ATTN),
    ("recurrence forgets to rescale l", "streaming.py",
     "l_new = l * alpha + p.sum(axis=1)", "l_new = l + p.sum(axis=1)", ATTN),
    ("recurrence masks the diagonal", "streaming.py",
     "ks[None, :] <= qpos[:, None]", "ks[None, :] < qpos[:, None]", ATTN),
    # schedule.py: ownership, rotation and pair classes ("Lesson 8", sections 2 and 4)
    ("zig-zag back band not mirrored", "schedule.py",
     "return place if band < _front_bands(k) else P - 1 - place",
     "return place if band < _front_bands(k) else place", SCHED),
    ("ring turns the wrong way", "schedule.py",
     "return [(first - hop) % P for hop in range(P)]", "return [(first + hop) % P for hop in range(P)]", SCHED),
    ("causal walk drops the diagonal", "schedule.py",
     'elif kc == qc:\n                        kind = "diag"',
     'elif kc == qc:\n                        kind = "skip"', SCHED),
    ("diagonal pair classed as full", "schedule.py",
     "elif not causal or kc < qc:", "elif not causal or kc <= qc:", SCHED),
    ("striped split dealt contiguously", "schedule.py",
     "return {r: list(range(r, S, P)) for r in range(P)}",
     "return {r: list(range(r * (S // P), (r + 1) * (S // P))) for r in range(P)}", SCHED),
    ("full tile tested on its first key", "schedule.py",
     "f = int(np.sum(k1[None, :] <= q0[:, None]))", "f = int(np.sum(k0[None, :] <= q0[:, None]))", SCHED),
    ("skipped tile tested against its first query", "schedule.py",
     "sk = int(np.sum(k0[None, :] > q1[:, None]))", "sk = int(np.sum(k0[None, :] > q0[:, None]))", SCHED),
    # helix.py: round-robin KV append ("NVIDIA unveils Helix Parallelism", KV cache growth)
    ("append deals token by token", "helix.py",
     "return (n // block) % P", "return n % P", HELIX),
]


def _scratch_tree(dst):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "*.tmp*", "__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for f in ("conftest.py", "test_oracle_attention.py", "test_oracle_backward.py", "test_oracle_schedule.py",
              "test_oracle_helix.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), os.path.join(dst, "pytest.ini"))


def _run_pins(dst, files):
    env = dict(os.environ, PYTHONPATH=dst, PYTHONDONTWRITEBYTECODE="1")
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *files],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=600)
    return p.returncode, (p.stdout + p.stderr)[-1500:]


def _mutant(base, idx):
    name, fname, old, new, files = MUTATIONS[idx]
    dst = os.path.join(base, f"m{idx}")
    _scratch_tree(dst)
    path = os.path.join(dst, "oracle", fname)
    src = open(path).read()
    if src.count(old) != 1:
        return name, None, f"the text to mutate occurs {src.count(old)} times in {fname}"
    open(path, "w").write(src.replace(old, new))
    rc, tail = _run_pins(dst, files)
    return name, rc, tail


def test_unmutated_copy_passes_its_pins(tmp_path):
    dst = str(tmp_path / "control")
    _scratch_tree(dst)
    rc, tail = _run_pins(dst, ATTN + BWD + SCHED + HELIX)
    assert rc == 0, tail


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda i: _mutant(str(tmp_path), i), range(len(MUTATIONS))))
    survivors = [(name, rc, tail) for name, rc, tail in results if rc != 1]
    assert not survivors, "\n\n".join(f"{n}: rc={rc}\n{t}" for n, rc, t in survivors)
