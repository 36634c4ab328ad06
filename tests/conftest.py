import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


import pytest  # noqa: E402


def _lib_stale() -> bool:
    pkg = os.path.join(ROOT, "masked_flash_attention_attn_b200")
    lib = os.path.join(pkg, "libattn_b200.so")
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    srcs = [os.path.join(pkg, "csrc", f) for f in os.listdir(os.path.join(pkg, "csrc"))]
    srcs.append(os.path.join(ROOT, "include", "attn.h"))
    return any(os.path.getmtime(s) > t for s in srcs)


@pytest.fixture(scope="session")
def attn_lib():
    """The in-tree C-ABI library, (re)built with nvcc when missing or older than its sources."""
    if _lib_stale():
        from masked_flash_attention_attn_b200 import build
        build.build()
    import masked_flash_attention_attn_b200 as M
    return M
