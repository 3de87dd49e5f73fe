"""The whole forward from pinned host Q, K, V to pinned host O, with the copies
overlapped with the computation.

The batch is cut into chunks of one batch index and a group of heads, each a
contiguous block of the host tensors. Three CUDA streams run the chunks as a
pipeline: while chunk c is packed and its forward runs on the compute stream,
chunk c + 1's Q, K, V travel host->device on the upload stream and chunk
c - 1's O travels device->host on the download stream (the two directions use
separate copy engines). Events order each chunk's upload, compute and
download. The bias is a learned parameter and stays on the device.

Every step of the computation is the library's (binattn.pack,
binattn.forward_ws); this module only places the calls and the copies.
"""
from __future__ import annotations

import torch

from . import binattn


class HostPipeline:
    """Device buffers, streams and events for one shape [B, H, N, d], reused
    across calls: run() allocates nothing.

    heads_per_chunk: heads of one batch index per chunk (a divisor of H). A
    chunk's forward launches ceil(N / 256) * heads_per_chunk CTAs, so the
    default (H, or H / 2 when that still fills the device) keeps each launch
    near a whole wave while giving the copies several chunks to overlap.
    """

    def __init__(self, B: int, H: int, N: int, d: int, device=None, heads_per_chunk: int | None = None,
                 has_bias: bool = True):
        self.B, self.H, self.N, self.d = B, H, N, d
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        if heads_per_chunk is None:
            nsm = torch.cuda.get_device_properties(self.device).multi_processor_count
            pairs_per_head = -(-N // 256)
            heads_per_chunk = H
            while heads_per_chunk % 2 == 0 and (heads_per_chunk // 2) * pairs_per_head >= nsm // 2:
                heads_per_chunk //= 2
        if H % heads_per_chunk:
            raise ValueError(f"heads_per_chunk {heads_per_chunk} does not divide H = {H}")
        self.hc = heads_per_chunk
        W = (d + 31) // 32
        dev = self.device
        bf = torch.bfloat16
        hc = self.hc
        self.chunks = [(b, h0) for b in range(B) for h0 in range(0, H, hc)]
        # one set of device buffers per chunk (each allocation aligned, which
        # slices of whole [B, H, ...] tensors need not be)
        self.buf = []
        for _ in self.chunks:
            q = torch.empty((1, hc, N, d), dtype=bf, device=dev)
            self.buf.append(dict(q=q, k=torch.empty_like(q), v=torch.empty_like(q), o=torch.empty_like(q),
                                 qb=torch.empty((1, hc, N, W), dtype=torch.int32, device=dev),
                                 kb=torch.empty((1, hc, N, W), dtype=torch.int32, device=dev),
                                 aq=torch.empty((1, hc, N), dtype=torch.float32, device=dev),
                                 ak=torch.empty((1, hc, N), dtype=torch.float32, device=dev)))
        need = binattn.workspace_bytes(1, self.hc, N, d, has_bias)
        self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        # a head group's bias planes start h0 * N * N elements into the bias;
        # when that is not 16-byte aligned (N odd), the chunk reads an aligned
        # copy made on the compute stream
        self.bias_copy = (torch.empty((hc, N, N), dtype=bf, device=dev)
                          if has_bias and (hc * N * N * 2) % 16 else None)
        self.s_up = torch.cuda.Stream(dev)
        self.s_cmp = torch.cuda.Stream(dev)
        self.s_down = torch.cuda.Stream(dev)
        self.ev_in = [torch.cuda.Event() for _ in self.chunks]
        self.ev_out = [torch.cuda.Event() for _ in self.chunks]
        self.ev_done = torch.cuda.Event()

    def run(self, q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, bias: torch.Tensor | None,
            softmax_scale: float, o_h: torch.Tensor, stream=None) -> None:
        """o_h = forward(q_h, k_h, v_h) for pinned host tensors [B,H,N,d] bf16;
        bias [H,N,N] bf16 on the device or None. Asynchronous: the work is
        ordered after `stream` (default: the current stream), which waits for
        its end; synchronize that stream before reading o_h."""
        for t, name in ((q_h, "q"), (k_h, "k"), (v_h, "v"), (o_h, "o")):
            if t.device.type != "cpu" or not t.is_pinned() or t.dtype != torch.bfloat16:
                raise ValueError(f"{name} must be a pinned host bfloat16 tensor")
            if tuple(t.shape) != (self.B, self.H, self.N, self.d) or not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous [{self.B}, {self.H}, {self.N}, {self.d}]")
        caller = torch.cuda.current_stream(self.device) if stream is None else stream
        start = torch.cuda.Event()
        start.record(caller)
        hc = self.hc
        for c, (b, h0) in enumerate(self.chunks):
            sl = (slice(b, b + 1), slice(h0, h0 + hc))
            x = self.buf[c]
            with torch.cuda.stream(self.s_up):
                self.s_up.wait_event(start)
                x["q"].copy_(q_h[sl], non_blocking=True)
                x["k"].copy_(k_h[sl], non_blocking=True)
                x["v"].copy_(v_h[sl], non_blocking=True)
                self.ev_in[c].record(self.s_up)
            with torch.cuda.stream(self.s_cmp):
                self.s_cmp.wait_event(self.ev_in[c])
                binattn.pack(x["q"], x["qb"], x["aq"], self.s_cmp)
                binattn.pack(x["k"], x["kb"], x["ak"], self.s_cmp)
                bias_c = None if bias is None else bias[h0:h0 + hc]
                if bias_c is not None and bias_c.data_ptr() % 16:
                    if self.bias_copy is None:
                        raise ValueError("the bias is not 16-byte aligned")
                    self.bias_copy.copy_(bias_c)
                    bias_c = self.bias_copy
                binattn.forward_ws(x["qb"], x["kb"], x["aq"], x["ak"], bias_c, x["v"], softmax_scale,
                                   workspace=self.ws, out=x["o"], stream=self.s_cmp)
                self.ev_out[c].record(self.s_cmp)
            with torch.cuda.stream(self.s_down):
                self.s_down.wait_event(self.ev_out[c])
                o_h[sl].copy_(x["o"], non_blocking=True)
        self.ev_done.record(self.s_down)
        caller.wait_event(self.ev_done)
