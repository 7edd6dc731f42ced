"""Decode steps fed from host memory: a thin wrapper of the library's native
step executor (pa_stepper_* in include/pagedattn.h).

One ``step`` call runs, in C++, the host allocator's step for the batch, the
uploads of q|k|v and of the block tables and lengths on the executor's copy
stream, the decode with the append on the compute stream, and the download of
the output, with the transfers of neighbouring steps overlapped with the
kernels (see csrc/pa_stepper.cpp). This module only converts arguments.
"""

import ctypes

import torch

from . import binding


class HostFedDecoder:
    def __init__(self, alloc, k_cache, v_cache, batch, max_blocks, max_len, out_dtype=None,
                 depth=2, partition=0, fused=True, stream=None):
        NB, H, S, D = k_cache.shape
        self.B, self.H, self.S, self.D, self.MB = batch, H, S, D, max_blocks
        self.fused = fused
        self.dtype = k_cache.dtype
        self.out_dtype = out_dtype or k_cache.dtype
        self.stream = stream or torch.cuda.current_stream(k_cache.device)
        self._keep = (alloc, k_cache, v_cache)  # the executor borrows these
        handle = ctypes.c_void_p()
        binding._check(binding.lib().pa_stepper_create(
            alloc._h, ctypes.c_void_p(k_cache.data_ptr()), ctypes.c_void_p(v_cache.data_ptr()),
            batch, H, D, S, NB, max_blocks, binding._DT[self.dtype], binding._DT[self.out_dtype],
            D ** -0.5, max_len, partition, int(fused), depth,
            ctypes.c_void_p(self.stream.cuda_stream), ctypes.byref(handle)), "pa_stepper_create")
        self._h = handle
        self._ids_key, self._ids = None, None
        self._step_no, self._max_len = ctypes.c_int64(), ctypes.c_int()

    def close(self):
        if self._h:
            binding.lib().pa_stepper_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def h2d_bytes(self):
        slots = 0 if self.fused else 8
        return 3 * self.B * self.H * self.D * torch.empty((), dtype=self.dtype).element_size() + \
            self.B * (slots + 4 * self.MB + 4)

    def d2h_bytes(self):
        return self.B * self.H * self.D * torch.empty((), dtype=self.out_dtype).element_size()

    def step(self, seq_ids, h_qkv):
        """Enqueues one decode step: every sequence in ``seq_ids`` grows by one
        token. ``h_qkv`` [3, batch, H, D] (q, k, v) in pinned host memory must stay
        unchanged until the step's upload has run. Returns (step number, longest
        sequence decoded)."""
        key = tuple(seq_ids)
        if key != self._ids_key:
            self._ids_key, self._ids = key, (ctypes.c_int64 * len(key))(*key)
        binding._check(binding.lib().pa_stepper_step(
            self._h, self._ids, ctypes.c_void_p(h_qkv.data_ptr()), ctypes.byref(self._step_no),
            ctypes.byref(self._max_len)), "pa_stepper_step")
        return self._step_no.value, self._max_len.value

    def output(self, step_no):
        """The output [batch, H, D] of a recent step (waits for its download)."""
        ptr = ctypes.c_void_p()
        binding._check(binding.lib().pa_stepper_output(self._h, step_no, ctypes.byref(ptr)),
                       "pa_stepper_output")
        n = self.d2h_bytes()
        buf = (ctypes.c_uint8 * n).from_address(ptr.value)
        return torch.frombuffer(bytearray(buf), dtype=self.out_dtype).view(self.B, self.H, self.D)

    def drain(self):
        """Makes the compute stream wait for every outstanding download."""
        binding._check(binding.lib().pa_stepper_drain(self._h), "pa_stepper_drain")
