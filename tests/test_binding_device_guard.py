"""The binding makes the tensors' device current around every native call.

The CUDA runtime launches on the calling thread's current device, and the
library keeps per-device state (kernel attributes, the allocation-free scratch
array), so a call for tensors on cuda:1 made while cuda:0 is current must
switch devices first.  Checked on the CPU with a fake library and a fake
device switch: no GPU is needed."""
import contextlib

import torch

from combine_warp_top_router_b200 import binding


class _FakeLib:
    def __init__(self, state):
        self.state = state

    def __getattr__(self, name):
        def fn(*args):
            self.state["calls"].append((name, self.state["current"], args))
            return 0
        return fn


def _patch(monkeypatch, current):
    state = {"current": current, "calls": []}

    @contextlib.contextmanager
    def fake_device(dev):
        old = state["current"]
        state["current"] = torch.device(dev).index
        try:
            yield
        finally:
            state["current"] = old

    monkeypatch.setattr(binding, "lib", lambda: _FakeLib(state))
    monkeypatch.setattr(binding.torch.cuda, "current_device", lambda: state["current"])
    monkeypatch.setattr(binding.torch.cuda, "device", fake_device)
    return state


def test_call_switches_to_the_tensors_device(monkeypatch):
    state = _patch(monkeypatch, current=0)
    assert binding._call("md_route_topk", torch.device("cuda", 1), 1, 2) == 0
    name, dev_during_call, args = state["calls"][-1]
    assert name == "md_route_topk" and dev_during_call == 1 and args == (1, 2)
    assert state["current"] == 0  # restored afterwards


def test_call_on_the_current_device_does_not_switch(monkeypatch):
    state = _patch(monkeypatch, current=3)
    binding._call("md_combine", torch.device("cuda", 3))
    assert state["calls"][-1][1] == 3


def test_every_compute_entry_point_goes_through_the_guard():
    # no binding function launches work through lib() directly
    import inspect
    src = inspect.getsource(binding)
    direct = [ln.strip() for ln in src.splitlines()
              if "lib().md_" in ln and "workspace_size" not in ln and "status_string" not in ln
              and "launch_count" not in ln and "memset_count" not in ln and "set_test_hooks" not in ln
              and "md_table1_row" not in ln and "md_pearson_from_sums" not in ln
              and "set_permute_path" not in ln and "set_layout_path" not in ln and "md_exchange_plan" not in ln]
    assert direct == []
