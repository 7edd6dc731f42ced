"""Decode steps fed from host memory, with transfers overlapped with kernels.

Each step of the decode loop ("vLLM KV Cache and PagedAttention Explained",
7단계 "전체 흐름 요약": the new token's K/V goes into the cache, then attention
reads the cached K/V) needs the step's q and new K/V, the block tables and the
lengths on the device, and its output back on the host. ``HostFedDecoder`` runs
those steps through the C ABI with the copies on a second CUDA stream and every
device and pinned host buffer ``depth`` sets deep, so the copies of step n+1
and the result copy of step n-1 run while the kernels of step n do:

  host          : pa_prepare_step(n) -> staging set n % depth
                  (after that set's upload of step n - depth has landed)
  copy stream   : wait compute(n - depth) ; upload q|k|v and tables|lengths ; record up(n)
  compute stream: wait up(n) ; pa_decode_append (or pa_kv_append + pa_decode) ; record compute(n)
  copy stream   : wait compute(n) ; download out(n) ; record down(n)

The KV cache is only touched on the compute stream, so steps stay in order.
Per step the host does one allocator call, two uploads, one decode call and
one download; the C calls go through ctypes with their arguments converted
once, so the host stays ahead of a ~200 us decode.
"""

import ctypes

import numpy as np
import torch

from . import binding


class HostFedDecoder:
    def __init__(self, alloc, k_cache, v_cache, batch, max_blocks, max_len, out_dtype=None,
                 depth=2, partition=0, fused=True):
        NB, H, S, D = k_cache.shape
        self.alloc, self.k_cache, self.v_cache = alloc, k_cache, v_cache
        self.B, self.H, self.S, self.D, self.MB = batch, H, S, D, max_blocks
        self.partition = partition
        self.fused = fused  # pa_decode_append (slots derived on the device) or two calls
        self.device = k_cache.device
        self.dtype = k_cache.dtype
        self.out_dtype = out_dtype or k_cache.dtype
        self.scale = D ** -0.5
        self.compute = torch.cuda.current_stream(self.device)
        self.copy = torch.cuda.Stream(self.device)
        ws = binding.pa_decode_workspace_bytes(batch, H, D, S, max_len, partition)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.device)
        dev, pin = dict(device=self.device), dict(pin_memory=True)
        meta_n = batch * max_blocks + batch
        self.sets = []
        for _ in range(depth):
            s = dict(
                h_slots=torch.empty(batch, dtype=torch.int64, **pin),
                h_meta=torch.empty(meta_n, dtype=torch.int32, **pin),  # tables | lengths
                h_out=torch.empty((batch, H, D), dtype=self.out_dtype, **pin),
                d_qkv=torch.empty((3, batch, H, D), dtype=self.dtype, **dev),
                d_slots=torch.empty(batch, dtype=torch.int64, **dev),
                d_meta=torch.empty(meta_n, dtype=torch.int32, **dev),
                d_out=torch.empty((batch, H, D), dtype=self.out_dtype, **dev),
                ev_up=torch.cuda.Event(), ev_compute=torch.cuda.Event(),
                ev_d2h=torch.cuda.Event(), used=False)
            s["h_tables"] = s["h_meta"][:batch * max_blocks].view(batch, max_blocks)
            s["h_lens"] = s["h_meta"][batch * max_blocks:]
            s["h_lens_np"] = s["h_lens"].numpy()
            s["d_tables"] = s["d_meta"][:batch * max_blocks].view(batch, max_blocks)
            s["d_lens"] = s["d_meta"][batch * max_blocks:]
            s["args"] = self._decode_args(s)
            self.sets.append(s)
        self._ids_key, self._ids = None, None
        self.n = 0

    def _decode_args(self, s):
        """pa_decode_append / pa_decode arguments of one buffer set, as ctypes values;
        the entry 'max_seq_len' is filled in per step."""
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        dt = binding._DT[self.dtype]
        q, k, v = s["d_qkv"][0], s["d_qkv"][1], s["d_qkv"][2]
        NB = self.k_cache.shape[0]
        common = dict(out=p(s["d_out"]), out_dt=binding._DT[self.out_dtype], q=p(q), k=p(k),
                      v=p(v), kc=p(self.k_cache), vc=p(self.v_cache), bt=p(s["d_tables"]),
                      lens=p(s["d_lens"]), ws=p(self.ws),
                      ws_bytes=self.ws.numel(), dt=dt, NB=NB)
        return common

    def h2d_bytes(self):
        slots = 0 if self.fused else 8
        return 3 * self.B * self.H * self.D * self.k_cache.element_size() + \
            self.B * (slots + 4 * self.MB + 4)

    def d2h_bytes(self):
        return self.B * self.H * self.D * torch.empty((), dtype=self.out_dtype).element_size()

    def _seq_ids(self, seq_ids):
        key = tuple(seq_ids)
        if key != self._ids_key:
            self._ids_key, self._ids = key, (ctypes.c_int64 * len(key))(*key)
        return self._ids

    def step(self, seq_ids, h_qkv):
        """Enqueues one decode step for ``seq_ids`` (each grows by one token).
        ``h_qkv`` [3, batch, H, D] holds q, k, v in pinned host memory and must stay
        unchanged until the step's upload has run. Returns (max length decoded,
        buffer set); the output is ``set["h_out"]`` once ``set["ev_d2h"]`` completes."""
        s = self.sets[self.n % len(self.sets)]
        lib = binding.lib()
        if s["used"]:
            s["ev_up"].synchronize()  # this set's previous upload has landed
        ids = self._seq_ids(seq_ids)
        rc = lib.pa_prepare_step(self.alloc._h, ids, len(ids), 1, self.MB,
                                 ctypes.c_void_p(s["h_slots"].data_ptr()),
                                 ctypes.c_void_p(s["h_tables"].data_ptr()),
                                 ctypes.c_void_p(s["h_lens"].data_ptr()))
        binding._check(rc, "pa_prepare_step")
        max_len = int(s["h_lens_np"].max())
        with torch.cuda.stream(self.copy):
            if s["used"]:
                self.copy.wait_event(s["ev_compute"])  # kernels of step n - depth read these
            s["d_qkv"].copy_(h_qkv, non_blocking=True)
            s["d_meta"].copy_(s["h_meta"], non_blocking=True)
            if not self.fused:
                s["d_slots"].copy_(s["h_slots"], non_blocking=True)
            s["ev_up"].record(self.copy)
        self.compute.wait_event(s["ev_up"])
        a = s["args"]
        st = ctypes.c_void_p(self.compute.cuda_stream)
        if self.fused:
            rc = lib.pa_decode_append(a["out"], a["out_dt"], a["q"], a["k"], a["v"], a["kc"],
                                      a["vc"], a["bt"], self.MB, a["lens"], self.scale, self.B,
                                      self.H, self.D, self.S, a["NB"], a["dt"], self.partition,
                                      max_len, a["ws"], a["ws_bytes"], st)
            binding._check(rc, "pa_decode_append")
        else:
            rc = lib.pa_kv_append(a["k"], a["v"], ctypes.c_void_p(s["d_slots"].data_ptr()),
                                  a["kc"], a["vc"], self.B, self.H, self.D, self.S, a["NB"],
                                  a["dt"], st)
            binding._check(rc, "pa_kv_append")
            rc = lib.pa_decode(a["out"], a["out_dt"], a["q"], a["kc"], a["vc"], a["bt"], self.MB,
                               a["lens"], self.scale, self.B, self.H, self.D, self.S, a["NB"],
                               a["dt"], self.partition, max_len, a["ws"], a["ws_bytes"], st)
            binding._check(rc, "pa_decode")
        s["ev_compute"].record(self.compute)
        with torch.cuda.stream(self.copy):
            self.copy.wait_event(s["ev_compute"])
            s["h_out"].copy_(s["d_out"], non_blocking=True)
            s["ev_d2h"].record(self.copy)
        s["used"] = True
        self.n += 1
        return max_len, s

    def drain(self):
        """Makes the compute stream wait for every outstanding result copy."""
        for s in self.sets:
            if s["used"]:
                self.compute.wait_event(s["ev_d2h"])
