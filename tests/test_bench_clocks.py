"""bench.py's reading of nvidia-smi clock samples, on CPU with a fake sample file: the
median SM clock under load, the max clock, and the throttle reasons seen active."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _DoneProcess:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _read(tmp_path, lines):
    path = tmp_path / "clocks.csv"
    path.write_text("".join(l + "\n" for l in lines))
    cs = bench.ClockSampler("GPU-00000000-0000-0000-0000-000000000000")
    cs.path, cs.proc = str(path), _DoneProcess()
    out = cs.stop()
    assert not path.exists()          # the sampler removes its file
    return out


# index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
def test_power_cap_is_reported_and_idle_samples_do_not_count(tmp_path):
    r = _read(tmp_path, ["0, 1965, 1965, 980.5, 0x4, Not Active, Not Active, Not Active, Active",
                         "0, 345, 1965, 120.0, 0x1, Not Active, Not Active, Not Active, Not Active",
                         "0, 1950, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active"])
    assert r["samples"] == 3
    assert r["sm_max_mhz"] == 1965.0
    assert r["sm_mhz"] == (1965.0 + 1950.0) / 2      # the idle 345 MHz sample is below half of max
    assert r["reasons"] == ["sw_power_cap"]


def test_slowdown_reasons_are_reported(tmp_path):
    r = _read(tmp_path, ["0, 1400, 1965, 700.0, 0x8, Active, Not Active, Not Active, Not Active",
                         "0, 1300, 1965, 650.0, 0x40, Not Active, Not Active, Active, Not Active"])
    assert r["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert r["sm_mhz"] == 1350.0


def test_no_samples_reads_as_none(tmp_path):
    assert _read(tmp_path, []) is None


class _Props:
    def __init__(self, uuid=None, domain=0, bus=0x3B, device=0):
        self.uuid, self.pci_domain_id, self.pci_bus_id, self.pci_device_id = uuid, domain, bus, device


def test_sampler_names_the_gpu_by_uuid_not_by_logical_index(monkeypatch):
    # With CUDA_VISIBLE_DEVICES=5, CUDA device 0 is the machine's GPU 5: nvidia-smi must
    # be given that GPU's UUID, never the logical index 0.
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "5")
    u = "4b1f6a2e-1c3d-4e5f-8a9b-0c1d2e3f4a5b"
    assert bench.nvsmi_device_id(_Props(uuid=u)) == "GPU-" + u
    assert bench.nvsmi_device_id(_Props(uuid="GPU-" + u)) == "GPU-" + u
    assert bench.nvsmi_device_id(_Props(uuid=None, bus=0x9A)) == "00000000:9a:00.0"
    seen = {}

    class _Popen:
        def __init__(self, cmd, **kw):
            seen["cmd"] = cmd

    monkeypatch.setattr(bench.subprocess, "Popen", _Popen)
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    cs = bench.ClockSampler(bench.nvsmi_device_id(_Props(uuid=u)))
    cs.start()
    os.unlink(cs.path)
    cmd = seen["cmd"]
    assert cmd[cmd.index("-i") + 1] == "GPU-" + u
    assert not any(a.startswith(("-lgc", "-ac", "-pm", "-rgc", "-r")) for a in cmd)   # read-only query
