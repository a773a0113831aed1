import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """FFN error margins: the worst cases against the tolerance, and every full-size case."""
    mod = sys.modules.get("gpu_util")
    if mod is None:
        return
    FFN_RESULTS, FFN_MAX_ABS, FFN_REL_L2 = mod.FFN_RESULTS, mod.FFN_MAX_ABS, mod.FFN_REL_L2
    if not FFN_RESULTS:
        return
    def frac(r):
        return max(r[1] / FFN_MAX_ABS, r[2] / FFN_REL_L2)
    worst = sorted(FFN_RESULTS, key=frac, reverse=True)
    full = [r for r in FFN_RESULTS if r[0].startswith("full:")]
    tr = terminalreporter
    tr.write_line(f"FFN margins: {len(FFN_RESULTS)} comparisons; tolerance max-abs {FFN_MAX_ABS:g}, "
                  f"rel-L2 {FFN_REL_L2:g}; largest fraction of it used: {frac(worst[0]):.2f}")
    for r in full + [w for w in worst[:6] if w not in full]:
        tr.write_line(f"  {r[0]}: max_abs={r[1]:.2e} rel_l2={r[2]:.2e} ({frac(r):.2f} of tolerance)")
