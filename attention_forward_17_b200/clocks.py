"""SM clock, power and clock-event reasons of one GPU, sampled while a timed
region runs (read queries only: nothing is set).  Used by the benchmark and by
the schedule search, so every timing that decides or reports a schedule
carries the clock it was taken at."""
from __future__ import annotations

import os
import statistics
import subprocess
import time


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU sampled while the
    timed region runs: NVML read queries from a background thread every 10 ms
    (nothing is set), or `nvidia-smi -lms 100` where NVML is unavailable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.01

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.rows = []
        self.source = None
        self.proc = None
        self.path = None
        self.thread = None

    def _nvml_loop(self, nv, handle, reason_fn, stop):
        smax = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap,
                "hw_power_brake": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown}
        while not stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(handle) / 1000.0
                rs = reason_fn(handle)
                self.rows.append(dict(sm=float(sm), smax=float(smax), power=pw,
                                      reasons={k for k, b in bits.items() if rs & b}))
            except Exception:
                pass
            stop.wait(self.PERIOD_S)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            handle = nv.nvmlDeviceGetHandleByIndex(self.gpu_index)
            reason_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop,
                                           args=(nv, handle, reason_fn, self.stop), daemon=True)
            self.thread.start()
            self.source = "nvml 10 ms"
            time.sleep(0.05)
            return self
        except Exception:
            self.thread = None
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "100"], stdout=self.out,
                stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi 100 ms"
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
                    self.rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                          reasons={n for n, v in zip(names, parts[5:9])
                                                   if v.lower() == "active"}))
                except ValueError:
                    continue
            os.unlink(self.path)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                    "source": self.source}
        load = [r for r in self.rows if r["power"] > 300] or self.rows
        reasons = set()
        for r in load:
            reasons |= r["reasons"]
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in self.rows),
                "power_w_max": max(r["power"] for r in self.rows),
                "samples": len(load), "reasons": sorted(reasons), "source": self.source}
