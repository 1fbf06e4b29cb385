"""CPU test of bench.py's clock sampler against a fake nvidia-smi: the sampler must be running
before the timed region starts, keep only the samples taken inside it, report throttle reasons
that were active there, and degrade to an empty summary when nvidia-smi is absent."""
import os
import time

import bench

LINE = "0, {sm}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {cap}"


def _fake_smi(tmp_path, body):
    path = tmp_path / "nvidia-smi"
    path.write_text("#!/bin/bash\n" + body + "\n")
    path.chmod(0o755)
    return str(tmp_path)


def test_samples_inside_the_region(tmp_path, monkeypatch):
    line = LINE.format(sm=1965, cap="Active")
    d = _fake_smi(tmp_path, f"while true; do echo '{line}'; sleep 0.05; done")
    monkeypatch.setenv("PATH", d + os.pathsep + os.environ["PATH"])
    t = time.monotonic()
    with bench.ClockSampler(0) as c:
        assert time.monotonic() - t < 2.0           # entered once the first sample arrived
        time.sleep(0.4)
    s = c.summary()
    assert s["window"] == "timed region"
    assert 4 <= s["samples"] <= 12
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_missing_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    with bench.ClockSampler(0) as c:
        pass
    s = c.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["reasons"] == []
