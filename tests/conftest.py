import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Largest parity errors seen by the GPU tests, per test file, and the full list as JSON
    when ATTN_PARITY_REPORT names a path."""
    try:
        from tests import gpu_util
    except Exception:  # pragma: no cover - the helpers import torch and the oracle
        return
    rep = gpu_util.REPORT
    if not rep:
        return
    import json
    path = os.environ.get("ATTN_PARITY_REPORT")
    if path:
        with open(path, "w") as fh:
            json.dump(rep, fh, indent=0)
    tr = terminalreporter
    tr.section("parity (GPU vs float64 oracle)")
    by_file = {}
    for r in rep:
        f = r["test"].split("::")[0] or "?"
        a = by_file.setdefault(f, {"checks": 0, "n": 0, "max_abs_bf16_f16": 0.0, "max_abs_below_4": 0.0,
                                   "n_over_1e-2": 0, "n_at_or_above_4": 0, "max_abs_f32": 0.0})
        a["checks"] += 1
        a["n"] += r["n"]
        if r["dtype"] == "f32":
            a["max_abs_f32"] = max(a["max_abs_f32"], r["max_abs"])
        else:
            a["max_abs_bf16_f16"] = max(a["max_abs_bf16_f16"], r["max_abs"])
            a["max_abs_below_4"] = max(a["max_abs_below_4"], r["max_abs_below_4"])
            a["n_over_1e-2"] += r["n_over_1e-2"]
            a["n_at_or_above_4"] += r["n_at_or_above_4"]
    for f, a in sorted(by_file.items()):
        tr.write_line(f"{f}: {a['checks']} checks, {a['n']} elements; 16-bit max |err| "
                      f"{a['max_abs_bf16_f16']:.3g} ({a['max_abs_below_4']:.3g} where |exact| < 4), "
                      f"{a['n_over_1e-2']} above 1e-2, each within its bound; {a['n_at_or_above_4']} elements with "
                      f"|exact| >= 4; fp32 max |err| {a['max_abs_f32']:.3g}")
    for r in rep:
        if any(k in r["test"] for k in ("cfg1", "cfg2", "cfg3", "cfg4", "cfg5", "ring_cfg5")):
            tr.write_line(f"  {r['test']} [{r['what']}, {r['dtype']}]: n={r['n']} max|err|={r['max_abs']:.3g} "
                          f"n>1e-2={r['n_over_1e-2']}")
