"""The C-ABI library loads, exports every entry point include/q1m.h declares, and rejects bad
arguments on the host before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

from long_context_prefill_dca_b200 import build, q1m
from synth import configs as C

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "q1m.h")


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(q1m_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return q1m.library()


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(q1m.SIGNATURES), set(names) ^ set(q1m.SIGNATURES)


def test_version(lib):
    assert "sm_100a" in q1m.version()


# Tests that pass stand-in pointers (small integers, not device memory) to reach a check that
# follows the NULL check. With no GPU present the library cannot launch anything, so a check
# that went missing fails the test instead of touching memory; on a machine with a GPU they
# are skipped.
host_only = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="passes stand-in device pointers; host-only")


@host_only
@pytest.mark.parametrize("field,value,code", [
    ("dca_chunk", 1000, -2),         # c - w not a multiple of 128
    ("local_window", -1, -1),
    ("prefill_chunk", 100, -1),
    ("vs_force_local", 0, -1),       # sparse needs the diagonal kept
    ("vs_last_q", 65, -1),
    ("in_dtype", 7, -1),
])
def test_invalid_params_rejected_without_launch(lib, field, value, code):
    p = q1m.params(C.SMALL_SPARSE)
    setattr(p, field, value)
    w = C.SMALL_SPARSE
    st = lib.q1m_dca_sparse_prefill(256, 256, 256, 256, None, w.seq_len, w.n_q_heads, w.n_kv_heads,
                                    w.head_dim, ctypes.byref(p), 256, 1 << 40, None)
    assert st == code, (st, lib.q1m_last_error())
    assert lib.q1m_last_error().decode()


@host_only
def test_bad_shapes_rejected(lib):
    w = C.SMALL_SPARSE
    p = q1m.params(w)
    assert lib.q1m_workspace_bytes(w.seq_len, 6, 4, 128, ctypes.byref(p)) == 0     # 6 % 4
    assert lib.q1m_workspace_bytes(w.seq_len, 4, 2, 96, ctypes.byref(p)) == 0      # head_dim
    assert lib.q1m_workspace_bytes(0, 4, 2, 128, ctypes.byref(p)) == 0
    st = lib.q1m_dca_sparse_prefill(None, 1, 1, 1, None, w.seq_len, 4, 2, 128, ctypes.byref(p),
                                    256, 1 << 40, None)
    assert st == -1
    st = lib.q1m_dca_sparse_prefill(256, 256, 256, 256, None, w.seq_len, 4, 2, 128, ctypes.byref(p),
                                    256, 10, None)
    assert st == -3          # workspace too small
    # NULL device pointers: nothing here can reach a launch, whatever the order of the checks
    st = lib.q1m_dca_sparse_prefill(None, None, None, None, None, w.seq_len, 16, 2, 128,
                                    ctypes.byref(p), None, 1 << 40, None)
    assert st == -2          # 8 Q heads per KV head exceeds the estimator


def test_workspace_sizes_monotone(lib):
    small = q1m.workspace_bytes(C.L7B_128K.seq_len, 28, 4, 128, q1m.params(C.L7B_128K))
    big = q1m.workspace_bytes(C.L7B_1M.seq_len, 28, 4, 128, q1m.params(C.L7B_1M))
    assert 0 < small < big < 40 * 2**30


@host_only
def test_decode_validates_before_launch():
    """q1m_dca_decode rejects bad arguments on the host, before touching the device."""
    import ctypes
    from long_context_prefill_dca_b200 import q1m
    from synth import configs as C
    lib = q1m.library()
    w = C.SMALL_SPARSE.with_(vs_vertical=0, vs_slash=0)
    p = q1m.params(w)
    nb = q1m.dca_decode_scratch_bytes(w.n_q_heads, w.head_dim)
    assert nb > 0 and q1m.dca_decode_scratch_bytes(4, 96) == 0
    args = lambda pos, ld, hq, hkv, d, sc: (1, 1, 1, pos, 256, 256, ld, hq, hkv, d, ctypes.byref(p), 256,
                                            256, None, 256, sc, None)
    assert lib.q1m_dca_decode(*args(-1, 1024, 4, 2, 128, nb)) == -1            # bad position
    assert lib.q1m_dca_decode(*args(1024, 1024, 4, 2, 128, nb)) == -1          # pos beyond the cache
    assert lib.q1m_dca_decode(*args(10, 1000, 4, 2, 128, nb)) == -1            # ld_tokens % 128
    assert lib.q1m_dca_decode(*args(10, 1024, 16, 1, 128, nb)) == -2           # G > 8
    assert lib.q1m_dca_decode(*args(10, 1024, 4, 2, 128, nb - 1)) == -3        # scratch too small
    assert lib.q1m_dca_decode(None, 1, 1, 10, 256, 256, 1024, 4, 2, 128, ctypes.byref(p), 256, 256,
                              None, 256, nb, None) == -1                       # NULL pointer


@host_only
def test_chunk_range_validated():
    import ctypes
    from long_context_prefill_dca_b200 import q1m
    from synth import configs as C
    lib = q1m.library()
    w = C.SMALL_SPARSE
    p = q1m.params(w)
    args = (256, 256, 256, 256, None, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, ctypes.byref(p))
    assert lib.q1m_dca_sparse_prefill_chunks(*args, -1, 2, 256, 1 << 40, None) == -1
    assert lib.q1m_dca_sparse_prefill_chunks(*args, 3, 2, 256, 1 << 40, None) == -1


def test_debug_mode_adds_guards_to_the_workspace():
    from long_context_prefill_dca_b200 import q1m
    from synth import configs as C
    w = C.SMALL_SPARSE
    args = (w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, q1m.params(w))
    base = q1m.workspace_bytes(*args)
    q1m.set_debug(True)
    try:
        assert q1m.debug_enabled()
        dbg = q1m.workspace_bytes(*args)
        assert dbg - base == 15 * 4096          # one guard after each of the 15 sparse-mode buffers
    finally:
        q1m.set_debug(False)
    assert q1m.workspace_bytes(*args) == base and not q1m.debug_enabled()
    with pytest.raises(q1m.Q1MError):
        q1m.debug_inject(99)
    q1m.debug_inject(-1)


def test_c_consumer_compiles_as_c_and_links(lib, tmp_path):
    """The header is valid C11 and the library links from C: a plain C program calls the
    GPU-free entry points and prints what the Python binding also sees."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(build.LIB)
    exe = str(tmp_path / "abi_consumer")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(root, "include"), os.path.join(root, "tests", "abi_consumer.c"),
                    "-L", libdir, "-l:" + os.path.basename(build.LIB), "-Wl,-rpath," + libdir,
                    "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.splitlines()
    got = {line.split(" ", 1)[0]: line.split(" ", 1)[1] for line in out}
    assert got["version"] == q1m.version()
    w = C.Workload(name="c", seq_len=1500, n_q_heads=4, n_kv_heads=2, head_dim=128,
                   in_dtype="bf16", rope_base=1e4, dca_chunk=384, local_window=128, yarn_s=2.0,
                   prefill_chunk=256, vs_vertical=20, vs_slash=70, vs_last_q=64, vs_force_local=8)
    for tag, ww in (("fixed", w), ("equal", w.with_(equal_cost_chunks=3))):
        ends = [e for _, e in q1m.prefill_bounds(ww)]
        assert got[tag].split() == [str(len(ends))] + [str(e) for e in ends], (tag, got[tag])
    assert got["too_many"] == "-3"
    p = q1m.params(w, "f32")
    assert int(got["workspace"]) == lib.q1m_workspace_bytes(1500, 4, 2, 128, ctypes.byref(p)) > 0
    assert int(got["host_workspace"]) == lib.q1m_host_workspace_bytes(1500, 4, 2, 128, ctypes.byref(p))
    assert int(got["decode_scratch"]) == q1m.dca_decode_scratch_bytes(4, 128) > 0
    assert got["null_status"] == "-1" and got["null_message"]
    # the binding's parameter block has the C layout, field by field
    assert int(got["sizeof_params"]) == ctypes.sizeof(q1m.Params)
    for name, _ in q1m.Params._fields_:
        assert int(got["offset_" + name]) == getattr(q1m.Params, name).offset, name
    assert {k[len("offset_"):] for k in got if k.startswith("offset_")} == \
        {n for n, _ in q1m.Params._fields_}


def _c_kind(decl: str) -> str:
    decl = decl.strip()
    if "*" in decl:
        return "ptr"
    base = decl.replace("const ", "").split()[0]
    return {"int": "i32", "int32_t": "i32", "q1m_status": "i32", "int64_t": "i64",
            "uint64_t": "u64", "size_t": "u64", "double": "f64", "void": "void"}[base]


def _ctypes_kind(t) -> str:
    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(t, "_type_") and t.__name__.startswith("LP_"):
        return "ptr"
    # size_t and uint64_t are the same 64-bit unsigned type on this ABI (LP64)
    assert ctypes.sizeof(ctypes.c_size_t) == ctypes.sizeof(ctypes.c_uint64) == 8
    return {ctypes.c_int: "i32", ctypes.c_int64: "i64", ctypes.c_uint64: "u64",
            ctypes.c_size_t: "u64", ctypes.c_double: "f64"}[t]


def test_binding_argument_kinds_match_the_header():
    """Every prototype in the header against the binding's ctypes signature: same number of
    arguments and, argument by argument, the same kind (32-bit int, 64-bit signed, 64-bit
    unsigned, double, pointer), and the same return kind."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    src = re.sub(r"#.*", "", src)
    protos = re.findall(r"([A-Za-z_][\w\s\*]*?)\b(q1m_\w+)\s*\(([^)]*)\)\s*;", src)
    assert len(protos) == len(q1m.SIGNATURES)
    for ret, name, params in protos:
        restype, argtypes = q1m.SIGNATURES[name]
        args = [a for a in params.split(",") if a.strip() and a.strip() != "void"]
        assert len(args) == len(argtypes), name
        for i, (a, t) in enumerate(zip(args, argtypes)):
            assert _c_kind(a) == _ctypes_kind(t), (name, i, a, t)
        assert _c_kind(ret) == _ctypes_kind(restype), (name, ret, restype)


def test_group_size_limits(lib):
    """Sparse mode takes at most 7 Q heads per KV head (the estimator's rows per group);
    dense mode has no such limit; decode takes at most 8."""
    w = C.SMALL_SPARSE
    p = q1m.params(w)
    assert lib.q1m_workspace_bytes(w.seq_len, 14, 2, 128, ctypes.byref(p)) > 0      # G = 7
    assert lib.q1m_workspace_bytes(w.seq_len, 16, 2, 128, ctypes.byref(p)) == 0     # G = 8
    st = lib.q1m_dca_sparse_prefill(None, None, None, None, None, w.seq_len, 16, 2, 128,
                                    ctypes.byref(p), None, 1 << 40, None)
    assert st == -2 and "7 Q heads" in lib.q1m_last_error().decode()
    pd = q1m.params(w.with_(vs_vertical=0, vs_slash=0))
    assert lib.q1m_workspace_bytes(w.seq_len, 16, 2, 128, ctypes.byref(pd)) > 0     # dense
    st = lib.q1m_dca_decode(None, None, None, 5, None, None, 128, 18, 2, 128, ctypes.byref(pd),
                            None, None, None, None, 1 << 20, None)
    assert st == -2, lib.q1m_last_error()


def test_header_limits_match_the_binding():
    """The size limits #defined in the header are the binding's constants."""
    src = open(HEADER).read()
    defs = dict(re.findall(r"#define\s+(Q1M_\w+)\s+(\d+)", src))
    assert int(defs["Q1M_MAX_CHUNK_QUERY_BLOCKS"]) == q1m.MAX_CHUNK_QUERY_BLOCKS
    assert int(defs["Q1M_NOALLOC_UNITS"]) == q1m.NOALLOC_UNITS
    assert int(defs["Q1M_NOALLOC_MAX_QUERY_BLOCKS"]) == q1m.NOALLOC_MAX_QUERY_BLOCKS
    # the static list holds the largest chunk it admits, and one block more does not fit
    units = lambda nqb: 3 * (nqb + 1) // 2 + 8
    assert units(q1m.NOALLOC_MAX_QUERY_BLOCKS) <= q1m.NOALLOC_UNITS < units(q1m.NOALLOC_MAX_QUERY_BLOCKS + 1)


def test_chunk_size_limit(lib):
    """A prefill chunk above Q1M_MAX_CHUNK_QUERY_BLOCKS query blocks is refused by the
    workspace query (0 bytes) and by the layer call before anything is launched; every device
    pointer is NULL, so a changed check order would be refused by the NULL check instead."""
    w = C.SMALL_DENSE_D128
    big = 128 * q1m.MAX_CHUNK_QUERY_BLOCKS
    ok = q1m.params(w.with_(seq_len=big, prefill_chunk=big))
    assert lib.q1m_workspace_bytes(big, 1, 1, 64, ctypes.byref(ok)) > 0
    p = q1m.params(w.with_(seq_len=big + 128, prefill_chunk=big + 128))
    assert lib.q1m_workspace_bytes(big + 128, 1, 1, 64, ctypes.byref(p)) == 0
    assert lib.q1m_host_workspace_bytes(big + 128, 1, 1, 64, ctypes.byref(p)) == 0
    st = lib.q1m_dca_sparse_prefill(None, None, None, None, None, big + 128, 1, 1, 64,
                                    ctypes.byref(p), None, 0, None)
    assert st == -2 and "exceeds" in lib.q1m_last_error().decode()
    # the same rows in chunks of the largest size are fine
    p2 = q1m.params(w.with_(seq_len=big + 128, prefill_chunk=big))
    assert lib.q1m_workspace_bytes(big + 128, 1, 1, 64, ctypes.byref(p2)) > 0
