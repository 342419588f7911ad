"""Raw cudaEvent_t handles for the per-kernel timing hook of moe_forward.

moe_dims.events takes 2*MOE_NUM_KERNELS event handles that the library records
on its stream right before and after each kernel. These helpers create such
handles and read their elapsed times through the CUDA runtime that torch has
already loaded in this process (measurement plumbing only)."""
from __future__ import annotations

import ctypes
import glob
import os
import sys

_rt = None


def cudart() -> ctypes.CDLL:
    global _rt
    if _rt is not None:
        return _rt
    import torch
    torch.cuda.init()
    cands = ["libcudart.so.12", "libcudart.so"]
    for p in sys.path:
        cands += sorted(glob.glob(os.path.join(p, "nvidia", "cuda_runtime", "lib", "libcudart.so*")))
    cands += sorted(glob.glob("/usr/local/cuda/lib64/libcudart.so*"))
    for c in cands:
        try:
            lib = ctypes.CDLL(c)
            lib.cudaEventCreate.argtypes = [ctypes.POINTER(ctypes.c_void_p)]
            lib.cudaEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p,
                                                 ctypes.c_void_p]
            lib.cudaEventDestroy.argtypes = [ctypes.c_void_p]
            lib.cudaEventRecord.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
            _rt = lib
            return lib
        except (OSError, AttributeError):
            continue
    raise RuntimeError("CUDA runtime library not found")


class KernelEvents:
    """One set of 2*n raw events; `.array` is what moe_dims.events points at."""

    def __init__(self, n_kernels: int):
        rt = cudart()
        self.n = n_kernels
        self.handles = []
        for _ in range(2 * n_kernels):
            h = ctypes.c_void_p()
            if rt.cudaEventCreate(ctypes.byref(h)) != 0:
                raise RuntimeError("cudaEventCreate failed")
            self.handles.append(h.value)
        self.array = (ctypes.c_void_p * (2 * n_kernels))(*self.handles)

    def elapsed_ms(self, i: int) -> float:
        """Device time of kernel i in ms (after the stream has been synchronised)."""
        out = ctypes.c_float()
        st = cudart().cudaEventElapsedTime(ctypes.byref(out), self.handles[2 * i],
                                           self.handles[2 * i + 1])
        if st != 0:
            raise RuntimeError(f"cudaEventElapsedTime failed ({st})")
        return float(out.value)

    def close(self):
        for h in self.handles:
            cudart().cudaEventDestroy(h)
        self.handles = []


def record(handle: int, stream: int) -> None:
    cudart().cudaEventRecord(handle, stream)
