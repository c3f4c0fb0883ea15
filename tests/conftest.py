import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


import pytest  # noqa: E402


@pytest.fixture(autouse=True)
def _error_words_clear(request, monkeypatch):
    """GPU tests: every PatchEmbed / PatchMerger handle a test creates ends with
    its device error word clear (a test that provokes an error reads, and so
    clears, the word itself): no pipeline wait gave up and, under the
    bounds-checking library, no access fell outside its buffer."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import torch
    from vlm_vision_patch_b200 import PatchEmbed, PatchMerger
    made = []
    for cls in (PatchEmbed, PatchMerger):
        def init(self, *a, _orig=cls.__init__, **k):
            _orig(self, *a, **k)
            made.append(self)
        monkeypatch.setattr(cls, "__init__", init)
    yield
    torch.cuda.synchronize()
    for obj in made:
        if getattr(obj, "h", None):
            assert obj.last_error() == 0, f"{type(obj).__name__}: device error word set"
