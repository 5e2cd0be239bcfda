"""Device-resident decode state on top of the C ABI.

A ``GqaSession`` does the same for the GQA route (qkn_gqa_append,
qkn_gqa_decode): the per-group expanded cache, the group weights, the raw
queries and a workspace.

A ``DecodeSession`` owns a paged cache, the key up-projection and norm
weights, the value up-projection (optional), the absorbed queries and a
decode workspace, and forwards to ``qkn_append``, ``qkn_absorb_query``,
``qkn_decode`` and ``qkn_decode_up``.  It moves host
arrays to the device and nothing else: all arithmetic runs in libqkn.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import (AK_CACHE, KERNEL_AUTO, Cache, Dims, GqaCache, absorb_query, append, append_absorb, decode, decode_up,
               gqa_append, gqa_decode, gqa_workspace_size, key_gram, decode_workspace_size, read_device_status,
               workspace_init)


def to_device(x, dtype: torch.dtype, device) -> torch.Tensor:
    if isinstance(x, torch.Tensor):
        return x.to(device=device, dtype=dtype).contiguous()
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype).contiguous()


class DecodeSession:
    def __init__(self, dims: Dims, num_blocks: int, device="cuda"):
        self.dims = dims
        self.device = torch.device(device)
        self.cache = Cache(dims, num_blocks, device=self.device)
        self.w_k = self.key_gram = self.gamma_q = self.gamma_k = self.gamma_qr = self.gamma_kr = None
        self.w_uv: Optional[torch.Tensor] = None
        self.q_tilde = self.a_q = self.q_rope_hat = None
        self.workspace: Optional[torch.Tensor] = None

    # ------------------------------------------------------------ weights
    def load_weights(self, w_k, gamma_q, gamma_k, gamma_qr, gamma_kr) -> None:
        f32, dev = torch.float32, self.device
        self.w_k = to_device(w_k, f32, dev)
        d = self.dims
        self.key_gram = torch.empty((d.num_groups, d.r_kv, d.r_kv), dtype=f32, device=dev)
        key_gram(d, self.w_k, self.key_gram)
        self.gamma_q = to_device(gamma_q, f32, dev)
        self.gamma_k = to_device(gamma_k, f32, dev)
        self.gamma_qr = to_device(gamma_qr, f32, dev)
        self.gamma_kr = to_device(gamma_kr, f32, dev)

    def load_value_weights(self, w_uv) -> None:
        """W^UV [H, r_kv, d_v], kept in the storage dtype (the fused merge reads it every step)."""
        self.w_uv = to_device(w_uv, self.dims.torch_dtype, self.device)

    # ------------------------------------------------------------ cache
    def append(self, c, k_rope_raw, slot, pos, chunk: int = 1 << 16) -> None:
        """Append tokens (host or device arrays) in chunks of ``chunk`` tokens."""
        dt, dev = self.dims.torch_dtype, self.device
        n = int(c.shape[0])
        for t0 in range(0, n, chunk):
            sl = slice(t0, min(n, t0 + chunk))
            append(self.dims, self.cache, to_device(c[sl], dt, dev), to_device(k_rope_raw[sl], dt, dev),
                   to_device(slot[sl], torch.int32, dev), to_device(pos[sl], torch.int32, dev),
                   self.w_k, self.key_gram, self.gamma_kr)

    # ------------------------------------------------------------ queries
    def absorb(self, q, q_rope, pos) -> None:
        """q [n_q, H, d_h], q_rope [n_q, H, d_R], pos [n_q] -> q~, a_q, q^R^ on the device.
        The output buffers are reused while the query count stays the same."""
        d, dt, dev = self.dims, self.dims.torch_dtype, self.device
        q = to_device(q, dt, dev)
        q_rope = to_device(q_rope, dt, dev)
        self.ensure_query_buffers(q.shape[0])
        absorb_query(d, q, q_rope, to_device(pos, torch.int32, dev), self.w_k, self.gamma_q, self.gamma_k,
                     self.gamma_qr, self.q_tilde, self.a_q, self.q_rope_hat)

    def prepare(self, c, k_rope_raw, slot, pos, q, q_rope, qpos) -> None:
        """A decode step's append and query absorption, in one launch where possible."""
        d, dt, dev = self.dims, self.dims.torch_dtype, self.device
        q = to_device(q, dt, dev)
        self.ensure_query_buffers(q.shape[0])
        append_absorb(d, self.cache, to_device(c, dt, dev), to_device(k_rope_raw, dt, dev),
                      to_device(slot, torch.int32, dev), to_device(pos, torch.int32, dev), q,
                      to_device(q_rope, dt, dev), to_device(qpos, torch.int32, dev), self.w_k, self.key_gram,
                      self.gamma_q,
                      self.gamma_k, self.gamma_qr, self.gamma_kr, self.q_tilde, self.a_q, self.q_rope_hat)

    def ensure_query_buffers(self, n_q: int) -> None:
        """Device buffers for q~, a_q and q^R^ of n_q query rows (kept while n_q stays the same)."""
        d, dt, dev = self.dims, self.dims.torch_dtype, self.device
        if self.q_tilde is None or self.q_tilde.shape[0] != n_q:
            self.q_tilde = torch.empty((n_q, d.num_heads, d.r_kv), dtype=dt, device=dev)
            self.a_q = torch.empty((n_q, d.num_heads), dtype=torch.float32, device=dev)
            self.q_rope_hat = torch.empty((n_q, d.num_heads, d.d_rope), dtype=dt, device=dev)

    # ------------------------------------------------------------ decode
    def ensure_workspace(self, batch: int, s_q: int) -> torch.Tensor:
        need = decode_workspace_size(self.dims, batch, s_q)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
            workspace_init(self.workspace)
        return self.workspace

    def decode(self, block_table, seq_lens, s_q: int, out=None, lse=None, ak_mode: int = AK_CACHE,
               kernel: int = KERNEL_AUTO, max_ctas: int = 0, head_tile: int = 0, wait_limit: int = 0,
               split_event=None, step_writes_only: bool = False, test_withhold_ak: bool = False, vis_end=None):
        d, dev = self.dims, self.device
        bt = to_device(block_table, torch.int32, dev)
        sl = to_device(seq_lens, torch.int32, dev)
        batch = bt.shape[0]
        ws = self.ensure_workspace(batch, s_q)
        if out is None:
            out = torch.empty((batch, s_q, d.num_heads, d.r_kv), dtype=d.torch_dtype, device=dev)
        if lse is None:
            lse = torch.empty((batch, s_q, d.num_heads), dtype=torch.float32, device=dev)
        decode(d, self.cache, self.q_tilde, self.a_q, self.q_rope_hat, bt, sl, s_q, ws, out, lse,
               ak_mode=ak_mode, kernel=kernel, max_ctas=max_ctas, head_tile=head_tile, wait_limit=wait_limit,
               split_event=split_event, step_writes_only=step_writes_only, test_withhold_ak=test_withhold_ak,
               vis_end=None if vis_end is None else to_device(vis_end, torch.int32, dev))
        return out, lse

    def decode_up(self, block_table, seq_lens, s_q: int, out_v=None, lse=None, ak_mode: int = AK_CACHE,
                  kernel: int = KERNEL_AUTO, max_ctas: int = 0, head_tile: int = 0, wait_limit: int = 0,
                  split_event=None, step_writes_only: bool = False):
        """The decode step with the value up-projection fused into the merge: o_v [batch, s_q, H, d_v]."""
        d, dev = self.dims, self.device
        if self.w_uv is None:
            raise RuntimeError("decode_up needs load_value_weights first")
        bt = to_device(block_table, torch.int32, dev)
        sl = to_device(seq_lens, torch.int32, dev)
        batch = bt.shape[0]
        ws = self.ensure_workspace(batch, s_q)
        if out_v is None:
            out_v = torch.empty((batch, s_q, d.num_heads, self.w_uv.shape[-1]), dtype=d.torch_dtype, device=dev)
        if lse is None:
            lse = torch.empty((batch, s_q, d.num_heads), dtype=torch.float32, device=dev)
        decode_up(d, self.cache, self.q_tilde, self.a_q, self.q_rope_hat, bt, sl, s_q, self.w_uv, ws, out_v, lse,
                  ak_mode=ak_mode, kernel=kernel, max_ctas=max_ctas, head_tile=head_tile, wait_limit=wait_limit,
                  split_event=split_event, step_writes_only=step_writes_only)
        return out_v, lse

    def device_status(self) -> int:
        return read_device_status(self.workspace)

    def clear_status(self) -> None:
        workspace_init(self.workspace)


def session_from_inputs(inp, device="cuda", dtype=None) -> DecodeSession:
    """Build a session from a seeded problem (an object with the fields of qkn_inputs.Inputs):
    weights loaded, every context token appended, queries absorbed."""
    wl = inp.wl
    dt = dtype if dtype is not None else (1 if wl.dtype == "bf16" else 0)
    dims = Dims(num_heads=wl.heads, num_groups=wl.groups, r_kv=wl.r_kv, d_h=wl.d_h, d_rope=wl.d_rope,
                eps=wl.eps, softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta, dtype=dt,
                block_size=wl.block_size)
    s = DecodeSession(dims, inp.num_blocks, device=device)
    s.load_weights(inp.w_k, inp.gamma_q, inp.gamma_k, inp.gamma_qr, inp.gamma_kr)
    s.load_value_weights(inp.w_uv)
    s.append(inp.c, inp.k_rope, inp.token_slots(), inp.token_positions())
    B, s_q = wl.batch, wl.s_q
    s.absorb(inp.q.reshape(B * s_q, wl.heads, wl.d_h), inp.q_rope.reshape(B * s_q, wl.heads, wl.d_rope),
             inp.query_positions().reshape(-1))
    return s


class GqaSession:
    """Device state of the GQA route: per-group keys and values expanded from the latent, the group weights
    W^UK_g, gamma_k[g], W^UV_g, the norm weights of the queries and RoPE key, the step's raw queries and a
    workspace."""

    def __init__(self, dims: Dims, num_blocks: int, d_v: int, device="cuda"):
        self.dims = dims
        self.device = torch.device(device)
        self.cache = GqaCache(dims, num_blocks, d_v, device=self.device)
        self.w_uk = self.gamma_k = self.w_uv = self.gamma_q = self.gamma_qr = self.gamma_kr = None
        self.q = self.q_rope = None
        self.workspace: Optional[torch.Tensor] = None

    def load_weights(self, w_uk, gamma_k, w_uv, gamma_q, gamma_qr, gamma_kr) -> None:
        """W^UK [g, r, d_h] and the gammas in fp32, W^UV [g, r, d_v] in the storage dtype."""
        f32, dev = torch.float32, self.device
        self.w_uk = to_device(w_uk, f32, dev)
        self.gamma_k = to_device(gamma_k, f32, dev)
        self.w_uv = to_device(w_uv, self.dims.torch_dtype, dev)
        self.gamma_q = to_device(gamma_q, f32, dev)
        self.gamma_qr = to_device(gamma_qr, f32, dev)
        self.gamma_kr = to_device(gamma_kr, f32, dev)

    def append(self, c, k_rope_raw, slot, pos, chunk: int = 1 << 16) -> None:
        dt, dev = self.dims.torch_dtype, self.device
        n = int(c.shape[0])
        for t0 in range(0, n, chunk):
            sl = slice(t0, min(n, t0 + chunk))
            gqa_append(self.dims, self.cache, to_device(c[sl], dt, dev), to_device(k_rope_raw[sl], dt, dev),
                       to_device(slot[sl], torch.int32, dev), to_device(pos[sl], torch.int32, dev), self.w_uk,
                       self.gamma_k, self.w_uv, self.gamma_kr)

    def set_queries(self, q, q_rope) -> None:
        """The step's raw queries: q [batch, s_q, H, d_h], q_rope [batch, s_q, H, d_R]."""
        dt, dev = self.dims.torch_dtype, self.device
        self.q = to_device(q, dt, dev)
        self.q_rope = to_device(q_rope, dt, dev)

    def ensure_workspace(self, batch: int, s_q: int) -> torch.Tensor:
        need = gqa_workspace_size(self.dims, self.cache.d_v, batch, s_q)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
            workspace_init(self.workspace)
        return self.workspace

    def decode(self, block_table, seq_lens, s_q: int, selection=None, max_ctas: int = 0, out_v=None, lse=None):
        """o_v [batch, s_q, H, d_v] and lse [batch, s_q, H]; ``selection`` [batch, s_q, g, k] for sparse."""
        d, dev = self.dims, self.device
        bt = to_device(block_table, torch.int32, dev)
        sl = to_device(seq_lens, torch.int32, dev)
        batch = bt.shape[0]
        ws = self.ensure_workspace(batch, s_q)
        if out_v is None:
            out_v = torch.empty((batch, s_q, d.num_heads, self.cache.d_v), dtype=d.torch_dtype, device=dev)
        if lse is None:
            lse = torch.empty((batch, s_q, d.num_heads), dtype=torch.float32, device=dev)
        sel = None if selection is None else to_device(selection, torch.int32, dev)
        gqa_decode(d, self.cache, self.q, self.q_rope, self.gamma_q, self.gamma_qr, bt, sl, s_q, ws, out_v, lse,
                   selection=sel, max_ctas=max_ctas)
        return out_v, lse

    def device_status(self) -> int:
        return read_device_status(self.workspace)

    def clear_status(self) -> None:
        workspace_init(self.workspace)


def gqa_session_from_inputs(inp, device="cuda") -> GqaSession:
    """A GQA-route session from a seeded problem of a tied-groups workload: group weights loaded, every
    context token expanded into the cache, the step's queries set."""
    wl = inp.wl
    dims = Dims(num_heads=wl.heads, num_groups=wl.groups, r_kv=wl.r_kv, d_h=wl.d_h, d_rope=wl.d_rope,
                eps=wl.eps, softmax_scale=wl.softmax_scale, rope_theta=wl.rope_theta,
                dtype=1 if wl.dtype == "bf16" else 0, block_size=wl.block_size)
    s = GqaSession(dims, inp.num_blocks, wl.d_v, device=device)
    w_uk, gamma_k, w_uv = inp.group_weights()
    s.load_weights(w_uk, gamma_k, w_uv, inp.gamma_q, inp.gamma_qr, inp.gamma_kr)
    s.append(inp.c, inp.k_rope, inp.token_slots(), inp.token_positions())
    s.set_queries(inp.q, inp.q_rope)
    return s

