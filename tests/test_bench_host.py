"""Host logic of bench.py that needs no GPU: the clock record of the timed region, read
through a fake NVML (the sampler only reads; nothing is set)."""
import sys
import time
import types

import pytest
import torch

import bench


class _FakeNvml(types.ModuleType):
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    class NVMLError(Exception):
        pass

    def __init__(self, clocks, reasons):
        super().__init__("pynvml")
        self.clocks, self.reasons, self.i, self.calls = clocks, reasons, 0, []

    def nvmlInit(self):
        self.calls.append("init")

    def nvmlShutdown(self):
        self.calls.append("shutdown")

    def nvmlDeviceGetHandleByUUID(self, uuid):
        assert uuid.startswith("GPU-")
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        v = self.clocks[min(self.i, len(self.clocks) - 1)]
        self.i += 1
        return v

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons[min(self.i, len(self.reasons)) - 1]


def _props():
    return types.SimpleNamespace(uuid="0000-1111", pci_domain_id=0, pci_bus_id=1,
                                 pci_device_id=0)


@pytest.fixture
def fake(monkeypatch):
    def make(clocks, reasons):
        nv = _FakeNvml(clocks, reasons)
        monkeypatch.setitem(sys.modules, "pynvml", nv)
        monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: _props())
        return nv
    return make


def test_nvml_region_records_clocks_and_reasons(fake):
    nv = fake([1965, 1965, 1950, 1965], [0, 0x4, 0, 0])
    reg = bench._NvmlRegion(0, period=0.001)
    reg.start()
    time.sleep(0.05)
    reg.stop()
    s = reg.summary()
    assert s["samples"] >= 4
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert nv.calls == ["init", "shutdown"]


def test_nvml_region_reports_thermal_reasons(fake):
    fake([1200] * 3, [0x40 | 0x8] * 3)
    reg = bench._NvmlRegion(0, period=0.001)
    reg.start()
    time.sleep(0.02)
    reg.stop()
    assert reg.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_without_nvml_the_summary_falls_back(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)      # import fails
    reg = bench._NvmlRegion(0)
    reg.start()
    reg.stop()
    assert reg.summary() is None and reg.error
    cs = bench.ClockSampler(0)
    cs.nvml, cs.lines = reg, ["0, 1965, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Active"]
    s = cs.summary()
    assert s["sm_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"] and s["samples"] == 1


def test_ks_permute_bmm_context_computes_the_factor():
    """The bench's permute + batched-GEMM context computes the same factor and gradients as
    the oracle (so its timing is of the same work)."""
    import numpy as np
    import torch

    import bench
    import oracle
    a, b, c, d, N = 3, 4, 5, 6, 7
    g = torch.Generator().manual_seed(0)
    w = torch.randn(a, d, b, c, generator=g, dtype=torch.float64)
    bias = torch.randn(a * c * d, generator=g, dtype=torch.float64)
    x = torch.randn(N, a * b * d, generator=g, dtype=torch.float64)
    G = torch.randn(N, a * c * d, generator=g, dtype=torch.float64)
    y, dx, dw, db = bench.ks_permute_bmm_step(x, G, w, bias, (a, b, c, d))
    ref = oracle.ks_backward(x.numpy(), w.numpy(), G.numpy())
    assert np.allclose(y.numpy(), oracle.ks_forward(x.numpy(), w.numpy(), bias.numpy()),
                       rtol=0, atol=1e-12)
    assert np.allclose(dx.numpy(), ref["dX"], rtol=0, atol=1e-12)
    assert np.allclose(dw.numpy(), ref["dw"], rtol=0, atol=1e-12)
    assert np.allclose(db.numpy(), ref["dbias"], rtol=0, atol=1e-12)
