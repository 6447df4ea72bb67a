"""CPU checks of the host-side helpers of the runner: the NUMA-local CPU binding computed
from NVML's affinity mask (a fake NVML here; reading it is all the helper does)."""
import os

import pytest

from mla_latent_kv_27_b200 import runner as R


class FakeNVML:
    def __init__(self, masks):
        self.masks = masks
        self.asked = None

    def nvmlDeviceGetCpuAffinity(self, handle, words):
        self.asked = words
        return self.masks


def _bind(monkeypatch, masks, allowed):
    nv = FakeNVML(masks)
    monkeypatch.setattr(R, "nvml_handle", lambda device: (nv, object()))
    monkeypatch.setattr(os, "sched_getaffinity", lambda pid: set(allowed))
    got = {}
    monkeypatch.setattr(os, "sched_setaffinity", lambda pid, cpus: got.setdefault("cpus", set(cpus)))
    res = R.bind_host_to_device("cuda:0")
    return res, got.get("cpus"), nv


def test_bind_uses_the_gpu_local_cpus(monkeypatch):
    # CPUs 1, 3 in word 0 and CPU 64 + 2 = 66 in word 1
    res, cpus, nv = _bind(monkeypatch, [0b1010, 0b100], allowed=range(128))
    assert res == [1, 3, 66] and cpus == {1, 3, 66}
    assert nv.asked == (os.cpu_count() + 63) // 64


def test_bind_keeps_only_cpus_the_process_may_use(monkeypatch):
    res, cpus, _ = _bind(monkeypatch, [0b1111], allowed=[2, 3, 9])
    assert res == [2, 3] and cpus == {2, 3}


def test_bind_leaves_affinity_alone_without_local_cpus(monkeypatch):
    res, cpus, _ = _bind(monkeypatch, [0b1], allowed=[5, 6])
    assert res is None and cpus is None


def test_bind_without_nvml_is_a_no_op(monkeypatch):
    def broken(device):
        raise RuntimeError("no NVML")
    monkeypatch.setattr(R, "nvml_handle", broken)
    called = []
    monkeypatch.setattr(os, "sched_setaffinity", lambda pid, cpus: called.append(cpus))
    assert R.bind_host_to_device("cuda:0") is None and not called
