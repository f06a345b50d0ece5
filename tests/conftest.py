import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session")
def cuda_lib():
    """The product library, loaded through its Python binding (GPU tests)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_attention_token_b200 as pa
    pa.load_library()
    return pa


def pytest_terminal_summary(terminalreporter):
    """Errors of every parity comparison the session made (GPU tests)."""
    from tests import parity
    if not parity.RECORDS:
        return
    tr = terminalreporter
    tr.write_sep("-", f"parity against the oracle ({len(parity.RECORDS)} comparisons; "
                      f"bar: max |err| <= {parity.MAX_ABS}, mean |err| <= {parity.MEAN_ABS})")
    for what, n, e in parity.RECORDS:
        tr.write_line(f"{what[:60]:<60} values {n:>9}  max {e['max_abs']:.2e}  mean {e['mean_abs']:.2e}  "
                      f"max_rel {e['max_rel']:.2e}  nan {e['nan']}")
