"""Receive buffers for the tensor-parallel QK-Norm with one rank per GPU.

In the paper's deployment every tensor-parallel rank is a process on its own
GPU: each rank publishes its scalar partial sums into every rank's receive
buffer (stores to peer memory over NVLink) and waits for the others' in its
own.  ``TpPeerExchange`` sets that up: it allocates this rank's receive
buffer (zeroed, ``qknorm_tp_recv_bytes(R, T)`` bytes), exports it as a CUDA IPC
handle, gathers every rank's handle over a ``torch.distributed`` process group
and opens the others' buffers in this process.  Its ``pointers()`` and
``next_epoch()`` go to ``qknorm_tp_layerwise(..., R=R, first_rank=rank)``
exactly as ``TpExchange``'s do in the single-GPU form; the library then uses
system-scope stores and loads for the exchange.

Every rank must call ``next_epoch`` once per call, in the same order, so that
all ranks of one call pass the same epoch; and pass the same blocks_per_rank
(0 on identical GPUs).  The IPC layer is injectable so that the handle
exchange can be tested on CPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _clib


class CudaIpc:
    """CUDA runtime IPC through cuda-python: device allocation, handles as
    64 bytes, opening and closing peer mappings."""

    def __init__(self):
        from cuda.bindings import runtime as rt  # imported only where CUDA is used
        self._rt = rt

    def _check(self, err, what: str):
        if err != self._rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"{what}: {self._rt.cudaGetErrorString(err)[1].decode()}")

    def alloc_zeroed(self, nbytes: int) -> int:
        err, ptr = self._rt.cudaMalloc(nbytes)
        self._check(err, "cudaMalloc")
        (err,) = self._rt.cudaMemset(ptr, 0, nbytes)
        self._check(err, "cudaMemset")
        (err,) = self._rt.cudaDeviceSynchronize()
        self._check(err, "cudaDeviceSynchronize")
        return int(ptr)

    def free(self, ptr: int):
        (err,) = self._rt.cudaFree(ptr)
        self._check(err, "cudaFree")

    def export(self, ptr: int) -> bytes:
        err, handle = self._rt.cudaIpcGetMemHandle(ptr)
        self._check(err, "cudaIpcGetMemHandle")
        return bytes(handle.reserved)

    def open(self, handle: bytes) -> int:
        h = self._rt.cudaIpcMemHandle_t()
        h.reserved = handle
        err, ptr = self._rt.cudaIpcOpenMemHandle(h, self._rt.cudaIpcMemLazyEnablePeerAccess)
        self._check(err, "cudaIpcOpenMemHandle")
        return int(ptr)

    def close(self, ptr: int):
        (err,) = self._rt.cudaIpcCloseMemHandle(ptr)
        self._check(err, "cudaIpcCloseMemHandle")


class TpPeerExchange:
    """This rank's receive buffer and the mapped buffers of the other ranks of
    an R-rank tensor-parallel group, one rank per process and GPU (the
    process's current CUDA device).  ``group`` is the process group of the R
    ranks (default: the world); rank r of the group is tensor-parallel rank r."""

    def __init__(self, R: int, T: int, group=None, ipc=None):
        n = _clib.load().qknorm_tp_recv_bytes(R, T)
        if n < 0:
            raise ValueError(f"invalid R={R} or T={T} for the exchange")
        if dist.get_world_size(group) != R:
            raise ValueError(f"the process group has {dist.get_world_size(group)} ranks, R = {R}")
        self.R, self.T = R, T
        self.rank = dist.get_rank(group)
        self._ipc = ipc if ipc is not None else CudaIpc()
        self._own = self._ipc.alloc_zeroed(max(n, 16))
        handles = [None] * R
        dist.all_gather_object(handles, self._ipc.export(self._own), group=group)
        self._opened = {}
        try:
            for r in range(R):
                if r != self.rank:
                    self._opened[r] = self._ipc.open(handles[r])
        except Exception:
            self.close()
            raise
        self._ptrs = [self._own if r == self.rank else self._opened[r] for r in range(R)]
        # every rank's buffer is zeroed and mapped before any rank publishes
        dist.barrier(group=group)
        self.epoch = 0

    def pointers(self):
        """recv[r] for r = 0 .. R-1: this rank's own buffer at its rank."""
        return list(self._ptrs)

    def next_epoch(self) -> int:
        self.epoch += 1
        if self.epoch >= 2 ** 32:
            raise RuntimeError("exchange epochs exhausted; make a new exchange")
        return self.epoch

    def close(self):
        """Unmaps the peers' buffers and frees this rank's (after every rank's
        last call has completed: the caller synchronizes first)."""
        for ptr in getattr(self, "_opened", {}).values():
            self._ipc.close(ptr)
        self._opened = {}
        if getattr(self, "_own", None):
            self._ipc.free(self._own)
            self._own = None
