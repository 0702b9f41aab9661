"""Host-side checks of the torch binding that need no GPU: the operands of a
call must share one CUDA device, and a stream passed in must belong to it
(the library reads every operand on the device it launches on)."""
from types import SimpleNamespace

import pytest
import torch

from selective_state_space_08_b200 import api


def _on(dev):
    return SimpleNamespace(device=torch.device(dev))


def test_one_device_accepts_one_device_and_skips_absent_operands():
    named = (("u", _on("cuda:1")), ("z", None), ("B", _on("cuda:1")), ("workspace", None))
    assert api._one_device(named) == torch.device("cuda:1")


def test_one_device_names_the_operand_on_another_device():
    named = (("u", _on("cuda:1")), ("delta", _on("cuda:1")), ("B", _on("cuda:0")))
    with pytest.raises(ValueError, match="B is on cuda:0"):
        api._one_device(named)


def test_stream_must_belong_to_the_operands_device():
    s = SimpleNamespace(device=torch.device("cuda:0"), cuda_stream=1234)
    assert api._stream(s, torch.device("cuda:0")).value == 1234
    with pytest.raises(ValueError, match="stream is on cuda:0"):
        api._stream(s, torch.device("cuda:1"))


def test_host_tensors_are_refused_where_device_tensors_are_expected():
    u = torch.zeros(1, 32, 8)
    with pytest.raises(ValueError, match="u must be a CUDA tensor"):
        api.scan_fwd(u, u, torch.zeros(32, 16), torch.zeros(1, 16, 8), torch.zeros(1, 16, 8))
