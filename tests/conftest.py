import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def gpu_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _device_status_stays_clear(request, monkeypatch):
    """GPU tests: every workspace the test makes (explicitly, or inside a
    binding call that was given none) must end the test with a clear device
    status word (no bounded wait ran out, no logit beyond the softmax bound,
    no index out of range).  Tests that provoke one of those read and clear
    it themselves."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import long_context_attention_csa_b200 as csa

    made = []
    orig = csa.workspace

    def recording(nbytes, device=None):
        t = orig(nbytes, device)
        made.append(t)
        return t

    monkeypatch.setattr(csa, "workspace", recording)
    yield
    for ws in made:
        assert csa.csa_check_status(ws) == (csa.CSA_OK, 0), "device status word set"


def pytest_terminal_summary(terminalreporter):
    """Worst bf16-ulp error of the parity comparisons that ran."""
    try:
        from parity import ULP_LOG
    except Exception:
        return
    if not ULP_LOG:
        return
    terminalreporter.write_sep("-", "parity: worst error in bf16 ulps of the reference (|ref| >= 1)")
    for what, ulps, ma, rel in sorted(ULP_LOG, key=lambda x: -x[1])[:12]:
        terminalreporter.write_line(f"{ulps:7.3f} ulp  max_abs {ma:.3e}  rel_l2 {rel:.3e}  {what}")
    terminalreporter.write_line(f"({len(ULP_LOG)} comparisons)")

