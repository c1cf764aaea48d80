"""Benchmark plumbing: process group, max-over-ranks timing, clock sampling,
L2 flush, and the algorithmic work of a verify step (for the roofline).

Nothing here computes the verify step itself.
"""
from __future__ import annotations

import json
import os
import statistics
import threading
import time

import numpy as np

# ------------------------------------------------------------------ algorithmic work
BYTES_PER_KEY = (512 + 64) * 2          # one c_kv + k_rope row (bf16)
BYTES_Q_ROW = (512 + 64) * 2            # one q_abs + q_rope row
BYTES_OUT_ROW = 512 * 2 + 4             # bf16 out row + fp32 lse


def attn_flops(cache_lens, depths, H: int) -> float:
    """QK over 576 plus PV over 512, visible (row, key) pairs only:
    2 * H * 1088 * (n * L_b + sum_i (depth_i + 1)) summed over requests."""
    total = 0.0
    for L, d in zip(cache_lens, depths):
        n = len(d)
        total += 2.0 * H * 1088 * (n * float(L) + float(np.sum(np.asarray(d) + 1)))
    return total


def attn_bytes(cache_lens, n: int, H: int) -> float:
    """KV read once per request, Q read once, out + lse written once."""
    kv = sum((float(L) + n) * BYTES_PER_KEY for L in cache_lens)
    return kv + len(cache_lens) * n * H * (BYTES_Q_ROW + BYTES_OUT_ROW)


def load_peaks(root: str) -> dict:
    """MEASURED_PEAKS.json when present, else the pool's earlier fallback figures."""
    p = os.path.join(root, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ distributed
def dist_env():
    """(rank, world, local_rank) from torchrun's environment (1 process if absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend: str, timeout_s: float = 120.0):
    import datetime

    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29511")
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank verifies its own batch (weak scaling): distinct seeds per rank."""
    return base_seed + 1000 * rank


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # pragma: no cover - no NVML on the CPU machine
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [v for k, v in self.REASONS.items() if self.reasons & k and v != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def clocks_rejected(c: dict) -> bool:
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    if any(r in bad for r in c.get("reasons", [])):
        return True
    if c.get("sm_mhz") and c.get("sm_max_mhz") and not c.get("reasons"):
        return c["sm_mhz"] < 0.5 * c["sm_max_mhz"]
    return False


# ------------------------------------------------------------------ L2 flush
class L2Flush:
    """Writes a buffer larger than the 126 MB L2 between timed repetitions."""

    def __init__(self, device, mbytes: int = 256):
        import torch
        self.buf = torch.empty(mbytes << 20, dtype=torch.uint8, device=device)

    def __call__(self):
        self.buf.fill_(1)


def blas_threads() -> tuple[int, str]:
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"]), str(info[0].get("internal_api"))
    except Exception:
        pass
    return len(os.sched_getaffinity(0)), "unknown"
