import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """The parity record of the run: per compared tensor max |err|, relative
    L2 error, the bound applied, and the elementwise allclose reading
    (atol 2e-2, rtol 1e-2) with its worst element."""
    parity = sys.modules.get("parity")
    records = getattr(parity, "RECORDS", None)
    if not records:
        return
    path = os.environ.get("SQA_PARITY_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(records, f, indent=1)
    n_ok = sum(r["allclose"] for r in records)
    scaled = [r for r in records if "*" in r["bound"]]
    tr = terminalreporter
    tr.section("parity record")
    tr.write_line(f"{len(records)} tensors compared; elementwise allclose (atol 2e-2, rtol 1e-2) holds for "
                  f"{n_ok}; {len(scaled)} used the scale-relative absolute bound")
    worst = sorted(records, key=lambda r: -r["rel_l2"])[:10]
    for r in worst + [r for r in scaled if r not in worst]:
        w = r["worst"] or {}
        tr.write_line(f"  {r['test'][:60]:60s} {r['what'][:24]:24s} max|err| {r['max_abs']:.2e} "
                      f"relL2 {r['rel_l2']:.2e} max|ref| {r['max_ref']:.2f} bound {r['bound']} "
                      f"allclose {r['allclose']} (worst {w.get('abs_err', 0):.2e} vs {w.get('allowed', 0):.2e})")
