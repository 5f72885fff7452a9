"""The C-ABI library loads on a machine without a GPU, exports every entry
point that include/tsenor.h declares, and rejects bad arguments on the host
before any CUDA call (no compute is run here)."""
import ctypes as C
import os
import re

import pytest

import sparse_mask_search_b200 as tsl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(tsenor_[a-z_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = tsl.lib()
    names = declared_functions()
    assert set(tsl.EXPORTS) <= set(names) | {"tsenor_last_error"}
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    L = tsl.lib()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert L.tsenor_status_string(code) != b"unknown status"
    assert L.tsenor_last_error() == b""


def test_largest_tau_is_accepted_up_to_the_documented_limit():
    # the header's TSENOR_MAX_TAU and the binding's copy agree; tau = 80 passes the
    # checks (the empty call returns before any launch), 80.5 does not
    text = open(os.path.join(ROOT, "include", "tsenor.h")).read()
    assert float(re.search(r"#define TSENOR_MAX_TAU ([0-9.]+)f", text).group(1)) == tsl.MAX_TAU == 80.0
    L = tsl.lib()
    assert _mask(L, rows=0, W=0, out=0, tau=80.0) == 0
    assert _mask(L, rows=0, W=0, out=0, tau=80.5) == -1


def _mask(L, W=1 << 12, dtype=1, rows=64, cols=64, N=2, M=4, tau=10.0, iters=5, sweeps=1, out=1 << 12):
    return L.tsenor_mask(W, dtype, rows, cols, N, M, tau, iters, sweeps, out, None)


@pytest.mark.parametrize("kw,code", [
    (dict(M=5), -3), (dict(M=128), -3), (dict(M=2), -3),
    (dict(N=0), -1), (dict(N=5), -1),
    (dict(rows=66), -2), (dict(cols=-4), -2),
    (dict(tau=0.0), -1), (dict(tau=float("nan")), -1), (dict(tau=float("inf")), -1),
    (dict(tau=80.5), -1), (dict(tau=200.0), -1),
    (dict(iters=0), -1), (dict(sweeps=-1), -1),
    (dict(dtype=7), -1),
    (dict(W=0), -1), (dict(W=(1 << 12) + 2), -1),
    (dict(out=0), -1), (dict(out=(1 << 12) + 4), -1),
])
def test_host_side_argument_errors(kw, code):
    assert _mask(tsl.lib(), **kw) == code


def test_empty_calls_do_nothing():
    L = tsl.lib()
    assert _mask(L, rows=0, W=0, out=0) == 0
    assert _mask(L, cols=0, W=0, out=0) == 0
    assert L.tsenor_plan(0, 0, 0, 32, 2, 4, 1.0, 3, 0, None) == 0
    assert L.tsenor_round(0, 0, 0, 32, 0, 2, 4, 1, 0, None) == 0
    assert L.tsenor_objective(0, 0, 0, 0, 0, 2, 4, 0, None) == 0


def test_other_entry_points_validate():
    L = tsl.lib()
    assert L.tsenor_plan(1 << 12, 1, 64, 64, 2, 4, 10.0, 5, 0, None) == -1        # no plan buffer
    assert L.tsenor_plan(1 << 12, 1, 64, 64, 2, 6, 10.0, 5, 1 << 12, None) == -3
    assert L.tsenor_round(1 << 12, 1 << 12, 1, 64, 64, 2, 4, -1, 1 << 12, None) == -1
    assert L.tsenor_objective(1 << 12, 1, 64, 62, 1 << 12, 2, 4, 1 << 12, None) == -2
    assert L.tsenor_error_count(None, None) == -1


def _warm(L, W=1 << 12, rows=64, cols=64, N=2, M=4, tau=10.0, iters=5, sweeps=1, tol=0.0, warm=0, pot=1 << 12,
          used=1 << 12, out=1 << 12):
    return L.tsenor_mask_warm(W, 1, rows, cols, N, M, tau, iters, sweeps, tol, warm, pot, used, out, None)


@pytest.mark.parametrize("kw,code", [
    (dict(tol=-1e-3), -1), (dict(tol=float("nan")), -1), (dict(tol=float("inf")), -1),
    (dict(warm=1, pot=0), -1), (dict(pot=(1 << 12) + 2), -1), (dict(used=(1 << 12) + 1), -1),
    (dict(out=0), -1), (dict(iters=0), -1), (dict(M=12), -3), (dict(cols=66), -2),
])
def test_warm_entry_points_validate(kw, code):
    L = tsl.lib()
    assert _warm(L, **kw) == code
    plan_kw = {k: v for k, v in kw.items() if k not in ("sweeps", "out")}
    if "out" not in kw:
        a = dict(W=1 << 12, rows=64, cols=64, N=2, M=4, tau=10.0, iters=5, tol=0.0, warm=0, pot=1 << 12,
                 used=1 << 12, out=1 << 12)
        a.update(plan_kw)
        assert L.tsenor_plan_warm(a["W"], 1, a["rows"], a["cols"], a["N"], a["M"], a["tau"], a["iters"], a["tol"],
                                  a["warm"], a["pot"], a["used"], a["out"], None) == code


def test_scores_entry_point_validates():
    L = tsl.lib()
    assert L.tsenor_mask_scores(1 << 12, 64, 64, 2, 4, 10.0, 5, 1, 0, None) == -1          # no mask buffer
    assert L.tsenor_mask_scores(1 << 12, 64, 62, 2, 4, 10.0, 5, 1, 1 << 12, None) == -2
    assert L.tsenor_mask_scores(0, 0, 64, 2, 4, 10.0, 5, 1, 0, None) == 0                   # empty


def test_host_entry_point_validates():
    L = tsl.lib()
    assert L.tsenor_mask_host(None, 1, 64, 64, 2, 4, 10.0, 5, 1, 1 << 12, None) == -1     # no W
    assert L.tsenor_mask_host(1 << 12, 1, 64, 64, 2, 4, 10.0, 5, 1, None, None) == -1     # no mask
    assert L.tsenor_mask_host(1 << 12, 1, 64, 62, 2, 4, 10.0, 5, 1, 1 << 12, None) == -2
    assert L.tsenor_mask_host(1 << 12, 1, 64, 64, 2, 6, 10.0, 5, 1, 1 << 12, None) == -3
    assert L.tsenor_mask_host(None, 1, 0, 64, 2, 4, 10.0, 5, 1, None, None) == 0          # empty


def test_warm_empty_calls_do_nothing():
    L = tsl.lib()
    assert _warm(L, rows=0, W=0, out=0, pot=0, used=0) == 0
    assert L.tsenor_plan_warm(0, 1, 0, 64, 2, 4, 10.0, 5, 0.0, 0, None, None, None, None) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(tsl, "_lib", None)
    monkeypatch.setattr(tsl, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        tsl.lib()
