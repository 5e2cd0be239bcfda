"""A whole decode step replayed as one CUDA graph.

Serving loops run the same step shape over and over: copy the step's new
tokens and queries in, append the tokens to the cache, absorb the queries,
decode, copy the result out.  ``DecodeStep`` captures that sequence once over
fixed buffers (pinned host buffers for the inputs and outputs, device buffers
for everything else) and replays it, so a step costs one graph launch instead
of a dozen API calls and copies.  Append and query absorption run as one
launch (qkn_append_absorb); the split-KV decode and its merge follow on the
same stream.  All arithmetic runs in libqkn.

Usage::

    step = DecodeStep(session, batch=B, s_q=1, max_blocks=M, n_tok=B)
    step.host_in["c"][:] = ...        # fill the pinned inputs (see NAMES)
    out, lse = step.run()             # pinned host outputs, valid after run() returns
"""
from __future__ import annotations

import torch

from . import AK_CACHE, KERNEL_AUTO, append_absorb, decode


class DecodeStep:
    # pinned host inputs of one step
    NAMES = ("c", "k_rope", "slot", "pos", "q", "q_rope", "qpos", "block_table", "seq_lens")

    def __init__(self, session, batch: int, s_q: int, max_blocks: int, n_tok: int, kernel: int = KERNEL_AUTO,
                 ak_mode: int = AK_CACHE, head_tile: int = 0):
        d = session.dims
        dt, dev, i32 = d.torch_dtype, session.device, torch.int32
        n_q = batch * s_q
        self.session, self.batch, self.s_q, self.kernel, self.ak_mode = session, batch, s_q, kernel, ak_mode
        self.head_tile = head_tile
        shapes = {
            "c": ((n_tok, d.r_kv), dt), "k_rope": ((n_tok, d.d_rope), dt),
            "slot": ((n_tok,), i32), "pos": ((n_tok,), i32),
            "q": ((n_q, d.num_heads, d.d_h), dt), "q_rope": ((n_q, d.num_heads, d.d_rope), dt),
            "qpos": ((n_q,), i32),
            "block_table": ((batch, max_blocks), i32), "seq_lens": ((batch,), i32),
        }
        # inputs and outputs are views of one byte buffer each (256-byte aligned fields), so that a
        # step moves them with one copy each way
        in_off, in_bytes = self._layout([shapes[k] for k in self.NAMES])
        self._host_in_buf = torch.zeros(in_bytes, dtype=torch.uint8, pin_memory=True)
        self._dev_in_buf = torch.zeros(in_bytes, dtype=torch.uint8, device=dev)
        self.host_in = self._views(self._host_in_buf, self.NAMES, shapes, in_off)
        self.dev_in = self._views(self._dev_in_buf, self.NAMES, shapes, in_off)
        oshapes = {"out": ((batch, s_q, d.num_heads, d.r_kv), dt), "lse": ((batch, s_q, d.num_heads), torch.float32)}
        out_off, out_bytes = self._layout([oshapes["out"], oshapes["lse"]])
        self._host_out_buf = torch.zeros(out_bytes, dtype=torch.uint8, pin_memory=True)
        self._dev_out_buf = torch.zeros(out_bytes, dtype=torch.uint8, device=dev)
        dv = self._views(self._dev_out_buf, ("out", "lse"), oshapes, out_off)
        hv = self._views(self._host_out_buf, ("out", "lse"), oshapes, out_off)
        self.out, self.lse = dv["out"], dv["lse"]
        self.host_out = (hv["out"], hv["lse"])
        session.ensure_query_buffers(n_q)
        self.workspace = session.ensure_workspace(batch, s_q)
        self.graph = None
        self.h2d_bytes = in_bytes
        self.d2h_bytes = out_bytes

    @staticmethod
    def _layout(fields):
        offs, pos = [], 0
        for shape, dtype in fields:
            offs.append(pos)
            n = int(torch.Size(shape).numel()) * torch.empty((), dtype=dtype).element_size()
            pos += (n + 255) // 256 * 256
        return offs, pos

    @staticmethod
    def _views(buf, names, shapes, offs):
        out = {}
        for name, off in zip(names, offs):
            shape, dtype = shapes[name]
            n = int(torch.Size(shape).numel()) * torch.empty((), dtype=dtype).element_size()
            out[name] = buf[off:off + n].view(dtype).view(shape)
        return out

    def _body(self) -> None:
        s, d, di = self.session, self.session.dims, self.dev_in
        self._dev_in_buf.copy_(self._host_in_buf, non_blocking=True)
        append_absorb(d, s.cache, di["c"], di["k_rope"], di["slot"], di["pos"], di["q"], di["q_rope"], di["qpos"],
                      s.w_k, s.key_gram, s.gamma_q, s.gamma_k, s.gamma_qr, s.gamma_kr, s.q_tilde, s.a_q,
                      s.q_rope_hat)
        decode(d, s.cache, s.q_tilde, s.a_q, s.q_rope_hat, di["block_table"], di["seq_lens"], self.s_q,
               self.workspace, self.out, self.lse, ak_mode=self.ak_mode, kernel=self.kernel, head_tile=self.head_tile,
               step_writes_only=True)
        self._host_out_buf.copy_(self._dev_out_buf, non_blocking=True)

    def capture(self) -> None:
        """Run the step once eagerly (first-call setup in the library), then capture it."""
        stream = torch.cuda.Stream(device=self.session.device)
        stream.wait_stream(torch.cuda.current_stream(self.session.device))
        with torch.cuda.stream(stream):
            self._body()
        stream.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream, capture_error_mode="relaxed"):
            self._body()
        torch.cuda.current_stream(self.session.device).wait_stream(stream)

    def run(self):
        """Replay the step on the current stream and wait for it; returns the pinned (out, lse)."""
        if self.graph is None:
            self.capture()
        self.graph.replay()
        torch.cuda.current_stream(self.session.device).synchronize()
        return self.host_out
