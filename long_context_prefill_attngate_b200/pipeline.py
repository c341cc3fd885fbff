"""Prefill of a layer that lives in host memory, with the PCIe copies
overlapped with the GPU work.

Every step of the path is independent per KV-head group (the gate, the mask
and the attention of a query head only read its own rows and its KV head),
so the layer is processed group by group on three CUDA streams: the copy-in
stream brings group c's Q/K/V to the device while the compute stream runs
gate -> TopK mask -> sparse attention on group c-1 and the copy-out stream
returns group c-2's O.  The result is identical to one whole-layer call of
each entry point (same kernels, same per-head arithmetic); only the order of
the copies changes.  Host tensors must be pinned for the copies to overlap.
"""
from __future__ import annotations

from . import _binding as B


class HostPrefill:
    """Device buffers for one layer shape, reused across calls."""

    def __init__(self, Bsz: int, Hq: int, Hkv: int, S: int, d: int, d_gate: int, device="cuda",
                 k_maxmin: bool = False):
        torch = B._torch()
        self.shape = (Bsz, Hq, Hkv, S, d)
        self.g = Hq // Hkv
        self.nb = -(-S // B.BLOCK)
        self.k_maxmin = k_maxmin
        dk = 2 * d if k_maxmin else d
        bf16 = torch.bfloat16
        self.q = torch.empty((Bsz, Hq, S, d), dtype=bf16, device=device)
        self.k = torch.empty((Bsz, Hkv, S, d), dtype=bf16, device=device)
        self.v = torch.empty((Bsz, Hkv, S, d), dtype=bf16, device=device)
        self.o = torch.empty((Bsz, Hq, S, d), dtype=bf16, device=device)
        self.wq = torch.empty((Hq, d, d_gate), dtype=bf16, device=device)
        self.wk = torch.empty((Hkv, dk, d_gate), dtype=bf16, device=device)
        self.scores = torch.empty((Bsz, Hq, self.nb, self.nb), dtype=torch.float32, device=device)
        self.mask = torch.empty((Bsz, Hq, self.nb, self.nb), dtype=torch.uint8, device=device)
        sub = B.seer_shape(1, self.g, 1, S, d)
        self.ws = torch.empty(B.seer_workspace_bytes(B.SEER_CALL_GATE_SCORES, sub), dtype=torch.uint8,
                              device=device)
        self.streams = [torch.cuda.Stream(device=device) for _ in range(3)]

    def run(self, hq, hk, hv, hwq, hwk, ho, density: float = 0.1, rope_theta: float = 5e5,
            force_first: bool = True, force_diag: bool = True):
        """Q/K/V/W from pinned host tensors -> O into the pinned host tensor ho.
        Work is ordered after everything already queued on the current
        stream, and the current stream waits for the last copy back."""
        torch = B._torch()
        Bsz, Hq, Hkv, S, d = self.shape
        g, nb = self.g, self.nb
        cur = torch.cuda.current_stream()
        s_in, s_c, s_out = self.streams
        start = torch.cuda.Event()
        start.record(cur)
        for s in self.streams:
            s.wait_event(start)
        with torch.cuda.stream(s_in):
            self.wq.copy_(hwq, non_blocking=True)
            self.wk.copy_(hwk, non_blocking=True)
        done_out = None
        for b in range(Bsz):
            for kvh in range(Hkv):
                h0, h1 = kvh * g, (kvh + 1) * g
                with torch.cuda.stream(s_in):
                    self.q[b, h0:h1].copy_(hq[b, h0:h1], non_blocking=True)
                    self.k[b, kvh].copy_(hk[b, kvh], non_blocking=True)
                    self.v[b, kvh].copy_(hv[b, kvh], non_blocking=True)
                    arrived = torch.cuda.Event()
                    arrived.record(s_in)
                s_c.wait_event(arrived)
                q = self.q[b:b + 1, h0:h1]
                k = self.k[b:b + 1, kvh:kvh + 1]
                v = self.v[b:b + 1, kvh:kvh + 1]
                sc = self.scores[b:b + 1, h0:h1]
                mk = self.mask[b:b + 1, h0:h1]
                o = self.o[b:b + 1, h0:h1]
                B.seer_gate_scores(q, k, self.wq[h0:h1], self.wk[kvh:kvh + 1], rope_theta=rope_theta, scores=sc,
                                   workspace=self.ws, stream=s_c, k_maxmin=self.k_maxmin)
                B.seer_block_mask(sc, "topk", density=density, force_first=force_first, force_diag=force_diag,
                                  mask=mk, stream=s_c, Hkv=1, d=d)
                B.seer_block_sparse_prefill(q, k, v, mk, o=o, stream=s_c)
                computed = torch.cuda.Event()
                computed.record(s_c)
                s_out.wait_event(computed)
                with torch.cuda.stream(s_out):
                    ho[b, h0:h1].copy_(self.o[b, h0:h1], non_blocking=True)
                    done_out = torch.cuda.Event()
                    done_out.record(s_out)
        cur.wait_event(done_out)
        return ho
