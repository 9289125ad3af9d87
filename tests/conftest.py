import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_terminal_summary(terminalreporter):
    """Errors of every checked GPU output, as written (no bf16 slack)."""
    try:
        import parity
    except ImportError:
        return
    if not parity.REPORT:
        return
    import json
    tr = terminalreporter
    tr.write_sep("-", "parity vs the fp64 oracle (errors as written, no bf16 slack)")
    agg = {}
    for r in parity.REPORT:
        kind = "lse" if "over_1e-3" in r else ("bf16" if r["bf16"] else "fp32")
        a = agg.setdefault((r["case"], kind), {"checks": 0, "max_abs": 0.0, "over": 0, "over_ge2": 0})
        a["checks"] += 1
        a["max_abs"] = max(a["max_abs"], r["max_abs"])
        a["over"] += r.get("over_1e-2", r.get("over_1e-3", 0))
        a["over_ge2"] += r.get("over_1e-2_at_abs_ref_ge_2", 0)
    tr.write_line("case | output | checks | max abs err | entries over the bound | of them at |oracle| >= 2")
    for (case, kind), a in sorted(agg.items()):
        tr.write_line(f"{case} | {kind} | {a['checks']} | {a['max_abs']:.3e} | {a['over']} | "
                      f"{a['over_ge2'] if kind != 'lse' else '-'}")
    path = os.environ.get("PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            for r in parity.REPORT:
                f.write(json.dumps(r) + "\n")
