"""The binding's checks on caller-supplied output buffers and workspaces: the library writes
through raw pointers, so anything but an exact match is refused before a call is made."""
import pytest
import torch

from exact_io_aware_93_b200 import api

CPU = torch.device("cpu")


def test_exact_buffer_accepted():
    api.check_buffer("out", torch.empty(2, 8, 4, 64, dtype=torch.bfloat16), (2, 8, 4, 64), torch.bfloat16, CPU)


@pytest.mark.parametrize("t", [
    torch.empty(2, 8, 4, 32, dtype=torch.bfloat16),                      # smaller
    torch.empty(2, 8, 4, 64, dtype=torch.float16),                       # other dtype
    torch.empty(2, 8, 64, 4, dtype=torch.bfloat16).transpose(2, 3),      # not contiguous
    "not a tensor",
])
def test_mismatched_buffer_refused(t):
    with pytest.raises(ValueError):
        api.check_buffer("out", t, (2, 8, 4, 64), torch.bfloat16, CPU)


def test_buffer_on_another_device_refused():
    with pytest.raises(ValueError):
        api.check_buffer("lse", torch.empty(2, 4, 8), (2, 4, 8), torch.float32, torch.device("cuda", 0))


def test_scratch_checks():
    api.check_scratch("workspace", torch.empty(100, dtype=torch.uint8), CPU)
    api.check_scratch("workspace", torch.empty(25, dtype=torch.float32), CPU)   # any dtype
    with pytest.raises(ValueError):
        api.check_scratch("workspace", torch.empty(10, 10)[:, ::2], CPU)
    with pytest.raises(ValueError):
        api.check_scratch("workspace", torch.empty(10), torch.device("cuda", 0))


def test_checking_build_selected_by_environment(monkeypatch):
    from exact_io_aware_93_b200 import build as fabuild
    monkeypatch.delenv("FA_B200_CHECKS", raising=False)
    assert api.library_path() == fabuild.LIB_PATH
    monkeypatch.setenv("FA_B200_CHECKS", "1")
    assert api.library_path() == fabuild.CHECKS_LIB_PATH
