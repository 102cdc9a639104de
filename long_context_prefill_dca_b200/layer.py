"""Convenience wrappers over the q1m C ABI: device buffers from PyTorch, calls into libq1m.

``Layer`` runs the whole chunked-prefill layer (``q1m_dca_sparse_prefill``); ``Stages`` runs
the same kernels one stage at a time (RoPE/DCA views, estimator, selection, block masks,
block-sparse attention, LSE merge) so each can be checked on its own. Nothing here computes:
tensors are allocated and pointers passed.
"""
from __future__ import annotations

import torch

from . import q1m


def _r128(x: int) -> int:
    return (x + 127) // 128 * 128


class Layer:
    def __init__(self, w, out_dtype: str = "f32", device="cuda"):
        self.w = w
        self.p = q1m.params(w, out_dtype)
        self.out_dtype = torch.bfloat16 if out_dtype == "bf16" else torch.float32
        self.ws_bytes = q1m.workspace_bytes(w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, self.p)
        if self.ws_bytes == 0:
            raise q1m.Q1MError("q1m_workspace_bytes", -1, "invalid shape or parameters")
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)

    def __call__(self, q, k, v, out=None, lse=None, stream=None):
        w = self.w
        if out is None:
            out = torch.empty(w.seq_len, w.n_q_heads, w.head_dim, dtype=self.out_dtype, device=q.device)
        q1m.dca_sparse_prefill(q, k, v, out, lse, w.seq_len, w.n_q_heads, w.n_kv_heads,
                               w.head_dim, self.p, self.ws, self.ws_bytes, stream)
        return out

    def chunks(self, q, k, v, first, last, out, lse=None, stream=None):
        """Prefill chunks [first, last) only, on this layer's workspace: a prefill resumed at
        chunk granularity (chunks before `first` must have run on this layer already)."""
        w = self.w
        q1m.dca_sparse_prefill_chunks(q, k, v, out, lse, w.seq_len, w.n_q_heads, w.n_kv_heads,
                                      w.head_dim, self.p, first, last, self.ws, self.ws_bytes,
                                      stream)
        return out


class HostLayer:
    """The layer from host (pinned) buffers through q1m_dca_sparse_prefill_host."""

    def __init__(self, w, out_dtype: str = "f32", device="cuda"):
        self.w = w
        self.p = q1m.params(w, out_dtype)
        self.ws_bytes = q1m.host_workspace_bytes(w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, self.p)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)

    def __call__(self, q_h, k_h, v_h, out_h, lse_h=None, stream=None):
        w = self.w
        q1m.dca_sparse_prefill_host(q_h, k_h, v_h, out_h, lse_h, w.seq_len, w.n_q_heads,
                                    w.n_kv_heads, w.head_dim, self.p, self.ws, self.ws_bytes, stream)
        return out_h


class Stages:
    """Buffers for running the layer stage by stage (one prefill chunk at a time)."""

    def __init__(self, w, out_dtype: str = "f32", device="cuda"):
        self.w, self.dev = w, device
        self.p = q1m.params(w, out_dtype)
        n, hq, hkv, d = w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim
        self.ld_tokens = _r128(n)
        self.ld_rows = _r128(max(e - s0 for s0, e in q1m.prefill_bounds(w)))
        self.table = torch.empty(w.dca_chunk * d, dtype=torch.float32, device=device)
        self.k_rot = torch.zeros(hkv, self.ld_tokens, d, dtype=torch.int16, device=device)
        self.v16 = torch.zeros(hkv, self.ld_tokens, d, dtype=torch.int16, device=device)
        self.qv = torch.empty(3, hq, self.ld_rows, d, dtype=torch.int16, device=device)
        self.o_part = torch.empty(3, hq, self.ld_rows, d, dtype=torch.float32, device=device)
        self.lse_part = torch.empty(3, hq, self.ld_rows, dtype=torch.float32, device=device)
        self.attn_scratch = torch.empty(q1m.attn_scratch_bytes(0, self.ld_rows, hq, d) + 64,
                                        dtype=torch.uint8, device=device)
        q1m.rope_table(self.table, w.dca_chunk, d, w.rope_base)

    # the views are fp16 bit patterns held in int16 tensors
    @staticmethod
    def as_f16(t):
        return t.view(torch.float16)

    def keys(self, k, v, s0, e):
        w = self.w
        q1m.rope_dca_keys(k, v, s0, e, w.n_kv_heads, w.head_dim, self.p, self.table, self.k_rot,
                          self.v16, self.ld_tokens)

    def queries(self, q, s0, e):
        w = self.w
        q1m.rope_dca_queries(q, s0, e, w.n_q_heads, w.head_dim, self.p, self.table, self.qv,
                             self.ld_rows)

    def estimate(self, q, s0, e):
        w = self.w
        vert = torch.empty(w.n_q_heads, e, dtype=torch.float32, device=self.dev)
        slash = torch.empty(w.n_q_heads, e, dtype=torch.float32, device=self.dev)
        nb = q1m.vs_estimate_scratch_bytes(e, w.n_q_heads, w.n_kv_heads, w.head_dim)
        scratch = torch.empty(nb, dtype=torch.uint8, device=self.dev)
        q1m.vs_estimate(q, self.k_rot, self.ld_tokens, s0, e, w.n_q_heads, w.n_kv_heads,
                        w.head_dim, self.p, self.table, vert, slash, e, scratch, nb)
        return vert, slash

    def select(self, vert, slash, e):
        w = self.w
        nv, ns = min(w.vs_vertical, e), min(w.vs_slash, e)
        V = torch.empty(w.n_q_heads, max(nv, 1), dtype=torch.int32, device=self.dev)
        S = torch.empty(w.n_q_heads, ns, dtype=torch.int32, device=self.dev)
        q1m.vs_select(vert, slash, vert.stride(0), e, w.n_q_heads, self.p, V, S)
        return V[:, :nv], S

    def masks(self, V, S, s0, e):
        w = self.w
        nqb = (e - s0 + 127) // 128
        nkw = ((e + 127) // 128 + 31) // 32
        nv = min(w.vs_vertical, e)
        mask = torch.empty(w.n_q_heads, nqb, nkw, dtype=torch.int32, device=self.dev)
        resid = torch.empty(w.n_q_heads, nqb, max(nv, 1), dtype=torch.int32, device=self.dev)
        cnt = torch.empty(w.n_q_heads, nqb, 8, dtype=torch.int32, device=self.dev)
        Vc = V.contiguous() if nv else torch.empty(w.n_q_heads, 1, dtype=torch.int32, device=self.dev)
        q1m.vs_build_masks(Vc, S.contiguous(), s0, e, w.n_q_heads, self.p, mask, resid, cnt)
        return mask, resid[:, :, :nv] if nv else resid[:, :, :0], cnt

    def attn(self, s0, e, mask=None, resid=None, cnt=None):
        w = self.w
        if mask is not None and (resid is None or resid.shape[-1] == 0):
            resid = torch.empty(w.n_q_heads, mask.shape[1], 1, dtype=torch.int32, device=self.dev)
        q1m.block_sparse_attn(self.qv, self.ld_rows, self.k_rot, self.v16, self.ld_tokens,
                              mask, resid.contiguous() if resid is not None else None, cnt, s0, e,
                              w.n_q_heads, w.n_kv_heads, w.head_dim, self.p, self.o_part,
                              self.lse_part, self.attn_scratch, self.attn_scratch.numel())

    def merge(self, s0, e, out, lse=None):
        w = self.w
        q1m.lse_merge(self.o_part, self.lse_part, 3, self.ld_rows, s0, e, w.seq_len,
                      w.n_q_heads, w.head_dim, self.p.out_dtype, self.p, out, lse)

    def decode(self, q_tok, k_tok, v_tok, pos, out, lse=None):
        """One decode step: the token at `pos` (q [Hq][D], k, v [Hkv][D]) is appended to the
        cache and attends keys [0, pos]; out [Hq][D], lse [Hq] (natural log)."""
        w = self.w
        nb = q1m.dca_decode_scratch_bytes(w.n_q_heads, w.head_dim)
        if getattr(self, "_dec_scratch", None) is None or self._dec_scratch.numel() < nb:
            self._dec_scratch = torch.empty(nb, dtype=torch.uint8, device=self.dev)
        q1m.dca_decode(q_tok, k_tok, v_tok, pos, self.k_rot, self.v16, self.ld_tokens,
                       w.n_q_heads, w.n_kv_heads, w.head_dim, self.p, self.table, out, lse,
                       self._dec_scratch, nb)
