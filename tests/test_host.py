"""Host placement helper (io_aware_exact_22_b200.host): NVML's CPU-affinity mask decoded, limited
to the CPUs this process may use, and applied only inside the `near_gpu` block.  NVML is
replaced by a fake: nothing here needs a GPU or changes a GPU setting."""
import os
import types

import pytest
import torch

from io_aware_exact_22_b200 import host


class FakeNVML:
    def __init__(self, words, fail=None):
        self.words = words
        self.fail = fail
        self.bus_ids = []
        self.inits = self.shutdowns = 0

    def nvmlInit(self):
        if self.fail == "init":
            raise RuntimeError("no driver")
        self.inits += 1

    def nvmlShutdown(self):
        self.shutdowns += 1

    def nvmlDeviceGetHandleByPciBusId(self, bus_id):
        if self.fail == "handle":
            raise RuntimeError("not found")
        self.bus_ids.append(bus_id)
        return object()

    def nvmlDeviceGetCpuAffinity(self, handle, n):
        return self.words[:n] + [0] * max(0, n - len(self.words))


@pytest.fixture
def fake_props(monkeypatch):
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1B, pci_device_id=0)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda dev: props)
    return props


def _mask(cpus):
    words = [0] * (max(cpus) // 64 + 1)
    for c in cpus:
        words[c // 64] |= 1 << (c % 64)
    return words


def test_bits_to_cpus():
    assert host._bits_to_cpus([0b1011, 1]) == {0, 1, 3, 64}
    assert host._bits_to_cpus([]) == set()
    assert host._bits_to_cpus([0, 1 << 63]) == {127}


def test_local_cpus_limited_to_allowed(fake_props):
    allowed = sorted(os.sched_getaffinity(0))
    want = set(allowed[: max(1, len(allowed) // 2)])
    nv = FakeNVML(_mask(want | {4095}))  # a CPU outside the allowed set is dropped
    assert host.local_cpus(0, nv) == want
    assert nv.bus_ids == ["00000000:1b:00.0"]
    assert nv.inits == nv.shutdowns == 1


@pytest.mark.parametrize("fail", ["init", "handle"])
def test_local_cpus_unknown(fake_props, fail):
    assert host.local_cpus(0, FakeNVML([1], fail=fail)) is None


def test_local_cpus_disjoint(fake_props):
    allowed = os.sched_getaffinity(0)
    outside = max(allowed) + 1
    assert host.local_cpus(0, FakeNVML(_mask({outside}))) is None


def test_near_gpu_binds_and_restores(fake_props):
    before = os.sched_getaffinity(0)
    target = {min(before)}
    with host.near_gpu(0, FakeNVML(_mask(target))) as cpus:
        assert cpus == target
        assert os.sched_getaffinity(0) == target
    assert os.sched_getaffinity(0) == before


def test_near_gpu_no_op_when_unknown(fake_props):
    before = os.sched_getaffinity(0)
    with host.near_gpu(0, FakeNVML([1], fail="init")) as cpus:
        assert cpus is None
        assert os.sched_getaffinity(0) == before
    assert os.sched_getaffinity(0) == before
