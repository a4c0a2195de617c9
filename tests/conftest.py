import pathlib
import sys

ROOT = pathlib.Path(__file__).resolve().parents[1]
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

GOLDEN = ROOT / "tests" / "golden"


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libkronq.so")
    config.addinivalue_line("markers", "slow: CPU oracle runs of tens of seconds")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def cuda():
    """The CUDA device for -m gpu tests; libkronq must be built and loadable
    (no skip where a GPU is present: a missing library is a failure)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_quantization_02_b200 import abi
    abi.lib()
    return torch.device("cuda", 0)
