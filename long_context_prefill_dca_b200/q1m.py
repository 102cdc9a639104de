"""Python binding of the q1m C ABI (include/q1m.h): argument marshalling only.

Every function here forwards to the entry point of the same name in libq1m.so; all the work
runs in the library's CUDA kernels. PyTorch supplies device memory and streams. There is
no fallback: if the library is not built, or the GPU is not an sm_100a device, calls raise.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

Q1M_OK = 0
STATUS = {0: "Q1M_OK", -1: "Q1M_ERR_INVALID", -2: "Q1M_ERR_UNSUPPORTED", -3: "Q1M_ERR_WORKSPACE",
          -4: "Q1M_ERR_CUDA", -5: "Q1M_ERR_TIMEOUT", -6: "Q1M_ERR_RANGE"}
BF16, F32 = 0, 1
# size limits, as include/q1m.h defines them
MAX_CHUNK_QUERY_BLOCKS = 32768      # Q1M_MAX_CHUNK_QUERY_BLOCKS
NOALLOC_UNITS = 16384               # Q1M_NOALLOC_UNITS
NOALLOC_MAX_QUERY_BLOCKS = 10916    # Q1M_NOALLOC_MAX_QUERY_BLOCKS

c_i32, c_i64, c_u64, c_dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
c_size, c_vp, c_int = ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int


class Params(ctypes.Structure):
    _fields_ = [("in_dtype", c_i32), ("out_dtype", c_i32), ("rope_base", c_dbl),
                ("yarn_s", c_dbl), ("dca_chunk", c_i64), ("local_window", c_i64),
                ("vs_vertical", c_i32), ("vs_slash", c_i32), ("vs_last_q", c_i32),
                ("vs_force_local", c_i32), ("prefill_chunk", c_i64),
                ("equal_cost_chunks", c_i32)]


class Q1MError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}")
        self.status = status


PP = ctypes.POINTER(Params)
# name -> (restype, argtypes)
SIGNATURES = {
    "q1m_workspace_bytes": (c_size, [c_i64, c_int, c_int, c_int, PP]),
    "q1m_dca_sparse_prefill": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_int, c_int, c_int,
                                       PP, c_vp, c_size, c_vp]),
    "q1m_host_workspace_bytes": (c_size, [c_i64, c_int, c_int, c_int, PP]),
    "q1m_dca_sparse_prefill_host": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_int, c_int,
                                            c_int, PP, c_vp, c_size, c_vp]),
    "q1m_rope_table": (c_int, [c_vp, c_i64, c_int, c_dbl, c_vp]),
    "q1m_rope_dca_keys": (c_int, [c_vp, c_vp, c_i64, c_i64, c_int, c_int, PP, c_vp, c_vp, c_vp,
                                  c_i64, c_vp]),
    "q1m_rope_dca_queries": (c_int, [c_vp, c_i64, c_i64, c_int, c_int, PP, c_vp, c_vp, c_i64,
                                     c_vp]),
    "q1m_vs_estimate_scratch_bytes": (c_size, [c_i64, c_int, c_int, c_int]),
    "q1m_vs_estimate": (c_int, [c_vp, c_vp, c_i64, c_i64, c_i64, c_int, c_int, c_int, PP, c_vp,
                                c_vp, c_vp, c_i64, c_vp, c_size, c_vp]),
    "q1m_vs_select_scratch_bytes": (c_size, [c_i64, c_int]),
    "q1m_vs_select": (c_int, [c_vp, c_vp, c_i64, c_i64, c_int, PP, c_vp, c_vp, c_vp, c_size,
                              c_vp]),
    "q1m_vs_build_masks": (c_int, [c_vp, c_vp, c_i64, c_i64, c_int, PP, c_vp, c_vp, c_vp, c_vp]),
    "q1m_attn_scratch_bytes": (c_size, [c_i64, c_i64, c_int, c_int]),
    "q1m_block_sparse_attn": (c_int, [c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_i64,
                                      c_i64, c_int, c_int, c_int, PP, c_vp, c_vp, c_vp, c_size,
                                      c_vp]),
    "q1m_block_sparse_attn_noalloc": (c_int, [c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp,
                                              c_i64, c_i64, c_int, c_int, c_int, PP, c_vp, c_vp,
                                              c_vp]),
    "q1m_lse_merge": (c_int, [c_vp, c_vp, c_int, c_i64, c_i64, c_i64, c_i64, c_int, c_int, c_int,
                              PP, c_vp, c_vp, c_vp]),
    "q1m_attention_recall": (c_int, [c_vp, c_vp, c_i64, c_vp, c_vp]),
    "q1m_prefill_bounds": (c_i64, [c_i64, PP, c_vp, c_i64]),
    "q1m_dca_sparse_prefill_chunks": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_int, c_int,
                                              c_int, PP, c_i64, c_i64, c_vp, c_size, c_vp]),
    "q1m_dca_decode_scratch_bytes": (c_size, [c_int, c_int]),
    "q1m_dca_decode": (c_int, [c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_int, c_int, c_int, PP,
                               c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "q1m_status_poll": (c_int, [c_vp]),
    "q1m_set_deterministic": (c_int, [c_int]),
    "q1m_deterministic": (c_int, []),
    "q1m_set_debug": (c_int, [c_int]),
    "q1m_debug_enabled": (c_int, []),
    "q1m_debug_inject": (c_int, [c_int]),
    "q1m_last_error": (ctypes.c_char_p, []),
    "q1m_version": (ctypes.c_char_p, []),
    "q1m_set_wait_budget": (c_int, [c_u64]),
    "q1m_profile_enable": (c_int, [c_int]),
    "q1m_profile_read": (c_int, [ctypes.POINTER(c_dbl), ctypes.POINTER(c_i64)]),
    "q1m_launch_count": (c_u64, []),
    "q1m_selftest_wait_timeout": (c_int, [c_u64, c_vp]),
    "q1m_selftest_exp2": (c_int, [c_vp, c_vp, c_vp, c_vp, c_i64, c_vp]),
}

_LIB = None


def library_path() -> str:
    return _build.LIB


def library():
    """Load libq1m.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise Q1MError("library", -4, f"{path} is not built "
                           "(python -m long_context_prefill_dca_b200.build)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def params(w, out_dtype: str | None = None) -> Params:
    """q1m_params of a synth.configs.Workload (or any object with the same fields)."""
    od = out_dtype or getattr(w, "out_dtype", "f32")
    return Params(BF16 if w.in_dtype == "bf16" else F32, BF16 if od == "bf16" else F32,
                  float(w.rope_base), float(w.yarn_s), int(w.dca_chunk), int(w.local_window),
                  int(w.vs_vertical), int(w.vs_slash), int(w.vs_last_q), int(w.vs_force_local),
                  int(w.prefill_chunk), int(getattr(w, "equal_cost_chunks", 0)))


def ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_handle(stream=None) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _call(name: str, *args) -> int:
    lib = library()
    st = getattr(lib, name)(*args)
    if st != Q1M_OK:
        raise Q1MError(name, st, lib.q1m_last_error().decode())
    return st


# ---- entry points (same names and arguments as the C ABI) ---------------------------------
def workspace_bytes(n, hq, hkv, d, p: Params) -> int:
    return library().q1m_workspace_bytes(n, hq, hkv, d, ctypes.byref(p))


def host_workspace_bytes(n, hq, hkv, d, p: Params) -> int:
    return library().q1m_host_workspace_bytes(n, hq, hkv, d, ctypes.byref(p))


def dca_sparse_prefill(q, k, v, out, lse, n, hq, hkv, d, p: Params, ws, ws_bytes, stream=None):
    _call("q1m_dca_sparse_prefill", ptr(q), ptr(k), ptr(v), ptr(out), ptr(lse), n, hq, hkv, d,
          ctypes.byref(p), ptr(ws), ws_bytes, stream_handle(stream))


def dca_sparse_prefill_chunks(q, k, v, out, lse, n, hq, hkv, d, p: Params, first, last, ws, ws_bytes,
                              stream=None):
    _call("q1m_dca_sparse_prefill_chunks", ptr(q), ptr(k), ptr(v), ptr(out), ptr(lse), n, hq, hkv,
          d, ctypes.byref(p), int(first), int(last), ptr(ws), ws_bytes, stream_handle(stream))


def dca_sparse_prefill_host(q, k, v, out, lse, n, hq, hkv, d, p: Params, ws, ws_bytes,
                            stream=None):
    _call("q1m_dca_sparse_prefill_host", ptr(q), ptr(k), ptr(v), ptr(out), ptr(lse), n, hq, hkv,
          d, ctypes.byref(p), ptr(ws), ws_bytes, stream_handle(stream))


def rope_table(table, n_pos, d, base, stream=None):
    _call("q1m_rope_table", ptr(table), n_pos, d, float(base), stream_handle(stream))


def rope_dca_keys(k, v, s0, e, hkv, d, p: Params, table, k_rot, v16, ld_tokens, stream=None):
    _call("q1m_rope_dca_keys", ptr(k), ptr(v), s0, e, hkv, d, ctypes.byref(p), ptr(table),
          ptr(k_rot), ptr(v16), ld_tokens, stream_handle(stream))


def rope_dca_queries(q, s0, e, hq, d, p: Params, table, qv, ld_rows, stream=None):
    _call("q1m_rope_dca_queries", ptr(q), s0, e, hq, d, ctypes.byref(p), ptr(table), ptr(qv),
          ld_rows, stream_handle(stream))


def vs_estimate_scratch_bytes(e, hq, hkv, d) -> int:
    return library().q1m_vs_estimate_scratch_bytes(e, hq, hkv, d)


def vs_estimate(q, k_rot, ld_tokens, s0, e, hq, hkv, d, p: Params, table, vert, slash, ld,
                scratch, scratch_bytes, stream=None):
    _call("q1m_vs_estimate", ptr(q), ptr(k_rot), ld_tokens, s0, e, hq, hkv, d, ctypes.byref(p),
          ptr(table), ptr(vert), ptr(slash), ld, ptr(scratch), scratch_bytes,
          stream_handle(stream))


def vs_select(vert, slash, ld, e, hq, p: Params, V, S, scratch=None, scratch_bytes=0,
              stream=None):
    _call("q1m_vs_select", ptr(vert), ptr(slash), ld, e, hq, ctypes.byref(p), ptr(V), ptr(S),
          ptr(scratch), scratch_bytes, stream_handle(stream))


def vs_build_masks(V, S, s0, e, hq, p: Params, mask, resid, cnt, stream=None):
    _call("q1m_vs_build_masks", ptr(V), ptr(S), s0, e, hq, ctypes.byref(p), ptr(mask),
          ptr(resid), ptr(cnt), stream_handle(stream))


def attn_scratch_bytes(s0, e, hq, d) -> int:
    return library().q1m_attn_scratch_bytes(s0, e, hq, d)


def block_sparse_attn(qv, ld_rows, k_rot, v16, ld_tokens, mask, resid, cnt, s0, e, hq, hkv, d,
                      p: Params, o_part, lse_part, scratch, scratch_bytes, stream=None):
    _call("q1m_block_sparse_attn", ptr(qv), ld_rows, ptr(k_rot), ptr(v16), ld_tokens, ptr(mask),
          ptr(resid), ptr(cnt), s0, e, hq, hkv, d, ctypes.byref(p), ptr(o_part), ptr(lse_part),
          ptr(scratch), scratch_bytes, stream_handle(stream))


def block_sparse_attn_noalloc(qv, ld_rows, k_rot, v16, ld_tokens, mask, resid, cnt, s0, e, hq,
                              hkv, d, p: Params, o_part, lse_part, stream=None):
    _call("q1m_block_sparse_attn_noalloc", ptr(qv), ld_rows, ptr(k_rot), ptr(v16), ld_tokens,
          ptr(mask), ptr(resid), ptr(cnt), s0, e, hq, hkv, d, ctypes.byref(p), ptr(o_part),
          ptr(lse_part), stream_handle(stream))


def lse_merge(o_part, lse_part, n_parts, ld_rows, s0, e, n, hq, d, out_dtype, p, out, lse,
              stream=None):
    _call("q1m_lse_merge", ptr(o_part), ptr(lse_part), n_parts, ld_rows, s0, e, n, hq, d,
          out_dtype, ctypes.byref(p) if p is not None else None, ptr(out), ptr(lse),
          stream_handle(stream))


def attention_recall(lse_sparse, lse_dense, recall, stream=None) -> None:
    _call("q1m_attention_recall", ptr(lse_sparse), ptr(lse_dense), lse_sparse.numel(), ptr(recall),
          stream_handle(stream))


def dca_decode_scratch_bytes(hq, d) -> int:
    return int(library().q1m_dca_decode_scratch_bytes(hq, d))


def dca_decode(q, k, v, pos, k_rot, v16, ld_tokens, hq, hkv, d, p, table, out, lse, scratch,
               scratch_bytes, stream=None) -> None:
    _call("q1m_dca_decode", ptr(q), ptr(k), ptr(v), int(pos), ptr(k_rot), ptr(v16), int(ld_tokens),
          hq, hkv, d, ctypes.byref(p), ptr(table), ptr(out), ptr(lse), ptr(scratch),
          int(scratch_bytes), stream_handle(stream))


def prefill_bounds(w) -> list[tuple[int, int]]:
    """(s0, e) of every prefill chunk of workload w, as the library's driver loop runs them
    (host computation; no GPU needed)."""
    n = int(w.seq_len)
    cap = n // 128 + 2
    ends = (c_i64 * cap)()
    p = params(w)
    m = library().q1m_prefill_bounds(n, ctypes.byref(p), ends, cap)
    if m < 0:
        raise Q1MError("q1m_prefill_bounds", int(m), library().q1m_last_error().decode())
    out, s0 = [], 0
    for e in ends[:m]:
        out.append((s0, int(e)))
        s0 = int(e)
    return out


def last_error() -> str:
    """The calling thread's last error message from the library."""
    return library().q1m_last_error().decode()


def set_deterministic(on: bool) -> None:
    _call("q1m_set_deterministic", 1 if on else 0)


def deterministic() -> bool:
    return bool(library().q1m_deterministic())


def set_debug(on: bool) -> None:
    _call("q1m_set_debug", 1 if on else 0)


def debug_enabled() -> bool:
    return bool(library().q1m_debug_enabled())


def debug_inject(stage: str | int) -> None:
    _call("q1m_debug_inject", STAGES.index(stage) if isinstance(stage, str) else int(stage))


def status_poll(stream=None) -> int:
    return library().q1m_status_poll(stream_handle(stream))


def check_status(stream=None) -> None:
    st = status_poll(stream)
    if st != Q1M_OK:
        raise Q1MError("q1m_status_poll", st, library().q1m_last_error().decode())


def set_wait_budget(cycles: int) -> None:
    _call("q1m_set_wait_budget", cycles)


def selftest_wait_timeout(cycles: int, stream=None) -> int:
    return library().q1m_selftest_wait_timeout(cycles, stream_handle(stream))


STAGES = ["table", "keys", "queries", "estimate", "select", "masks", "attn", "merge", "decode"]


def profile_enable(on: bool = True) -> None:
    _call("q1m_profile_enable", 1 if on else 0)


def profile_read() -> dict:
    """{stage: (ms, launches)} accumulated since profile_enable()."""
    ms = (c_dbl * len(STAGES))()
    n = (c_i64 * len(STAGES))()
    _call("q1m_profile_read", ms, n)
    return {name: (ms[i], n[i]) for i, name in enumerate(STAGES)}


def launch_count() -> int:
    return int(library().q1m_launch_count())


def selftest_exp2(x, y_poly, y_mufu, y_ref, stream=None) -> None:
    _call("q1m_selftest_exp2", ptr(x), ptr(y_poly), ptr(y_mufu), ptr(y_ref), x.numel(),
          stream_handle(stream))


def version() -> str:
    return library().q1m_version().decode()
