"""Shared test helpers: tolerances and oracle comparisons of device results."""
import numpy as np
import torch

import oracle

# Tolerances (max |gpu - oracle| over the checked entries).
TOL_FP32 = 1e-5          # float32 path: out and lse
TOL_BF16_OUT = 2e-2      # bf16 in / fp32 accumulate: out (after the bf16 rounding of the output)
TOL_BF16_LSE = 1e-3      # bf16 path: lse


# Every parity check made through margin() is recorded here; tests/conftest.py
# prints the worst ratio of error to tolerance per check at the end of the run,
# so a log shows the headroom of each configuration and not only pass / fail.
MARGINS: list = []


def margin(quantity: str, err, tol, what: str = "") -> float:
    """Assert err <= tol for one parity check (max |gpu - reference| of
    `quantity`) and record it under the running test's id."""
    import os
    err = float(err)
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0].replace("tests/", "")
    name = test if (not what or what in test) else f"{test} {what}"
    MARGINS.append((name, quantity, err, float(tol)))
    assert err <= tol, f"{name}: max |{quantity} - reference| = {err:.3e} > {tol}"
    return err


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def oracle_rows(q, k, v, rows, scale, causal, **kw):
    return oracle.attention_rows(host(q), host(k), host(v), rows, scale=scale, causal=causal, **kw)


def check_rows(out, lse, rows, ref_out, ref_lse, tol_out, tol_lse, what=""):
    """out [B,S,Hq,D], lse [B,Hq,S] (device) against oracle results for `rows`."""
    rows = np.asarray(rows)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    o = host(out)[b, i, h, :]
    l = host(lse)[b, h, i]
    err_o = np.max(np.abs(o - ref_out))
    err_l = np.max(np.abs(l - ref_lse))
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l)), what
    margin("out", err_o, tol_out, what)
    margin("lse", err_l, tol_lse, what)
    return err_o, err_l


def need_cuda():
    import pytest
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for tests marked gpu")
