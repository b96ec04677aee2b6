"""Device buffers of one layer's recurrent state, allocated with torch, and
a step loop over the C ABI.  Marshalling only: the arithmetic is in
libbrs.so."""
from __future__ import annotations

import torch

from . import brs


class LayerState:
    """Stored state + residuals + statistics + workspace of one layer."""

    def __init__(self, layout: brs.Layout, device="cuda", perm=None):
        self.layout = layout
        self.device = torch.device(device)
        nbytes, aux, stats, ws = brs.state_bytes(layout)
        self.packed = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.aux = torch.zeros(max(aux, 16), dtype=torch.uint8, device=self.device)
        self.stats = torch.zeros(max(stats, 16), dtype=torch.uint8, device=self.device)
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=self.device)
        self.state32 = None            # FP32 state between write-backs (deferred write-back)
        self.prefill_ws = None         # chunked prefill: flag word + FP32 state between chunks
        self.perm = None
        if perm is not None:
            self.perm = torch.as_tensor(perm, dtype=torch.int16).contiguous().to(self.device)

    def pack(self, S: torch.Tensor, widths=None):
        """Store S (deterministic rounding).  The auxiliary buffer (error-
        feedback residuals or direction counters) is left as it is: zero()
        or aux.zero_() starts those from 0."""
        brs.state_pack(self.layout, S.contiguous(), self.perm, self.packed, self.workspace,
                       widths=widths)

    def unpack(self) -> torch.Tensor:
        L = self.layout
        S = torch.empty((L.B, L.H, L.d, L.d), dtype=torch.float32, device=self.device)
        brs.state_unpack(L, self.packed, self.perm, S, self.workspace)
        return S

    def zero(self):
        L = self.layout
        self.pack(torch.zeros((L.B, L.H, L.d, L.d), dtype=torch.float32, device=self.device))
        self.aux.zero_()
        self.stats.zero_()

    def step(self, wb: brs.WriteBack, t: int, q, k, v, beta, decay, o, packed_out=None):
        if wb.C > 1:
            # deferred write-back: the FP32 state between write-backs
            if self.state32 is None:
                self.state32 = torch.zeros(brs.decode_state32_bytes(self.layout) // 4, dtype=torch.float32,
                                           device=self.device)
            brs.decode_step_deferred(self.layout, wb, t, self.packed, self.aux, self.workspace, self.state32,
                                     self.perm, q, k, v, beta, decay, o)
            return self.packed
        out = self.packed if packed_out is None else packed_out
        brs.decode_step(self.layout, wb, t, self.packed, out, self.aux, self.stats,
                        self.workspace, self.perm, q, k, v, beta, decay, o)
        if packed_out is not None:
            self.packed, out = out, self.packed
        return out

    def prefill(self, wb: brs.WriteBack, step0: int, T: int, q, k, v, beta, decay, o, state_dump=None):
        """brs_chunk_prefill over T tokens (sequence-major inputs)."""
        if self.prefill_ws is None:
            self.prefill_ws = torch.zeros(brs.prefill_workspace_bytes(self.layout), dtype=torch.uint8,
                                          device=self.device)
        brs.chunk_prefill(self.layout, wb, step0, T, self.packed, self.aux, self.prefill_ws, self.perm,
                          q, k, v, beta, decay, o, state_dump=state_dump)

    def errors(self) -> int:
        fl = brs.fetch_errors(self.workspace)
        if self.prefill_ws is not None:
            fl |= brs.fetch_errors(self.prefill_ws)
        return fl
