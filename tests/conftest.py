import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def mla_lib():
    """Build (if needed) and load libmla.so through the package binding."""
    from head_latent_attention_attn_b200 import build as _build
    import head_latent_attention_attn_b200 as mla
    _build.build()
    return mla.lib()
