"""Host-side placement of pinned buffers for host <-> device copies.

A DMA copy between pinned host memory and a GPU runs at full PCIe bandwidth only when the
host pages sit on the NUMA node that the GPU's PCIe root hangs off; pages on the other socket
cross the inter-socket link.  `local_cpus` asks NVML (read-only query) which CPUs are close to
a CUDA device, and `near_gpu` runs a block with the calling thread bound to them, so that
pinned buffers allocated inside it are placed on the GPU's node.  The previous affinity is
restored on exit; copies issued later do not depend on it.
"""
from __future__ import annotations

import contextlib
import os


def _nvml():
    try:
        import pynvml  # nvidia-ml-py
    except ImportError:
        return None
    return pynvml


def _bits_to_cpus(words, word_bits: int = 64) -> set[int]:
    """CPU indices set in an NVML affinity mask (a list of unsigned words, lowest CPUs first)."""
    cpus = set()
    for w, word in enumerate(words):
        word = int(word)
        b = 0
        while word:
            if word & 1:
                cpus.add(w * word_bits + b)
            word >>= 1
            b += 1
    return cpus


def local_cpus(device: int, nvml=None) -> set[int] | None:
    """CPUs that NVML reports as closest to CUDA device `device` (torch numbering), limited to
    the CPUs this process may run on; None when NVML or the device's PCI id is unavailable, or
    when the two sets do not meet."""
    nvml = nvml if nvml is not None else _nvml()
    if nvml is None:
        return None
    try:
        import torch
        p = torch.cuda.get_device_properties(device)
        bus_id = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except Exception:
        return None
    try:
        nvml.nvmlInit()
    except Exception:
        return None
    try:
        h = nvml.nvmlDeviceGetHandleByPciBusId(bus_id)
        ncpu = os.cpu_count() or 1
        words = nvml.nvmlDeviceGetCpuAffinity(h, (ncpu + 63) // 64)
    except Exception:
        return None
    finally:
        try:
            nvml.nvmlShutdown()
        except Exception:
            pass
    cpus = _bits_to_cpus(words) & set(os.sched_getaffinity(0))
    return cpus or None


@contextlib.contextmanager
def near_gpu(device: int, nvml=None):
    """Binds the calling thread to `local_cpus(device)` for the duration of the block (no-op
    when they are unknown); yields the CPU set used, or None."""
    cpus = local_cpus(device, nvml)
    if not cpus:
        yield None
        return
    old = os.sched_getaffinity(0)
    os.sched_setaffinity(0, cpus)
    try:
        yield cpus
    finally:
        os.sched_setaffinity(0, old)
