"""The C-ABI library builds, loads and exports every function include/pa.h
declares (CPU only: no compute calls)."""
import ctypes

import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import build


def test_library_builds_and_exports_every_declared_symbol():
    build.build()
    lib = pa.lib()
    names = pa.header_functions()
    assert {"pa_decode", "pa_reshape_and_cache", "pa_copy_blocks", "pa_decode_workspace_size"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/pa.h but not exported"


def test_host_only_entry_points():
    lib = pa.lib()
    assert lib.pa_status_string(0) == b"PA_OK"
    assert lib.pa_status_string(2) == b"PA_ERR_UNSUPPORTED"
    # partition choice and workspace size are pure host functions
    assert pa.pa_decode_partition_size(8, 32, 8, 128, 64, 32768, 512) == 512
    assert pa.pa_decode_partition_size(4, 2, 2, 64, 16, 33, 0) == 48        # one partition
    assert pa.pa_decode_partition_size(64, 32, 32, 128, 16, 2048, 0) == 256  # one head per KV head
    assert pa.pa_decode_partition_size(4, 2, 2, 64, 16, 33, 24) == 0        # not a multiple of 16
    assert pa.pa_decode_partition_size(4, 32, 4, 128, 16, 100, 0) == 112    # group 8: one partition
    assert pa.pa_decode_partition_size(4, 32, 4, 128, 16, 8192, 0) == 512   # 512-token partitions
    assert pa.pa_decode_partition_size(4, 32, 4, 128, 64, 8192, 2048) == 2048  # 32 blocks of 64
    assert pa.pa_decode_partition_size(4, 32, 4, 128, 16, 8192, 1024) == 0     # > 32 blocks
    assert pa.pa_decode_partition_size(4, 24, 4, 128, 16, 100, 0) == 0      # group 6 unsupported
    n = pa.pa_decode_workspace_size(8, 32, 8, 128, 64, 32768, 512)
    parts = 32768 // 512
    assert n >= 8 * parts * 16 + 8 * 32 * parts * (8 + 128 * 4)
    assert lib.pa_decode_workspace_size(4, 2, 2, 96, 16, 33, 0) == 0        # head_dim 96


def test_reshape_rejects_bad_arguments_without_a_device():
    lib = pa.lib()
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 1, 2, 64, 16, 32, 0, None) == pa.PA_ERR_INVALID
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 1, 2, 96, 16, 32, 0, None) == pa.PA_ERR_UNSUPPORTED
    ptrs = (ctypes.c_void_p * 1)(None)
    assert lib.pa_copy_blocks(ptrs, 1, None, 1, 100, 32, None) == pa.PA_ERR_INVALID
    assert lib.pa_last_error() != b""


def test_shared_decode_host_checks_without_a_device():
    lib = pa.lib()
    plain = pa.pa_decode_workspace_size(64, 32, 8, 128, 16, 2048, 0)
    shared = pa.pa_decode_shared_workspace_size(64, 32, 8, 128, 16, 2048, 0)
    # one more partition of partials per sequence, the second entry words and the member lists
    parts = 2048 // 512
    assert shared >= plain + 64 * 32 * (8 + 128 * 4) + 64 * (parts + 1) * 16 + 2 * 64 * 4
    assert lib.pa_decode_shared_workspace_size(4, 2, 2, 96, 16, 33, 0) == 0
    # 8-bit cache: 512 tokens at every group size, head_dim 64 or 128
    assert pa.pa_decode_fp8_partition_size(64, 32, 32, 128, 16, 2048, 0) == 512
    assert pa.pa_decode_fp8_partition_size(256, 32, 8, 128, 16, 8192, 0) == 512
    assert pa.pa_decode_fp8_partition_size(8, 32, 8, 128, 64, 32768, 0) == 512
    assert pa.pa_decode_fp8_partition_size(8, 32, 8, 64, 16, 4096, 0) == 512
    assert pa.pa_decode_fp8_partition_size(8, 32, 8, 64, 32, 300, 0) == 320  # one partition
    assert pa.pa_decode_fp8_partition_size(8, 32, 8, 96, 16, 4096, 0) == 0
    # same partitions as pa_decode here (512 tokens), so the same workspace
    assert pa.pa_decode_fp8_workspace_size(256, 32, 8, 128, 16, 8192, 0) == pa.pa_decode_workspace_size(
        256, 32, 8, 128, 16, 8192, 0)
    assert 0 < pa.pa_decode_fp8_workspace_size(64, 32, 32, 128, 16, 2048, 0) < pa.pa_decode_workspace_size(
        64, 32, 32, 128, 16, 2048, 0)  # 512 against 256 tokens at one head per KV head: fewer slots
    # shared-prefix units: 16 blocks for grouped heads, as pa_decode otherwise
    assert pa.pa_decode_shared_partition_size(4, 32, 8, 128, 16, 8192, 0) == 256
    assert pa.pa_decode_shared_partition_size(4, 32, 32, 128, 16, 8192, 0) == 256
    assert pa.pa_decode_shared_partition_size(4, 32, 8, 128, 16, 100, 0) == 112
    assert pa.pa_decode_shared_partition_size(4, 32, 8, 128, 16, 8192, 512) == 512
    dummy = ctypes.c_void_p(256)
    args = [dummy, dummy, None, None, dummy, dummy, dummy, dummy]
    rest = [32, 8, 128, 16, 64, 4096, 1024, ctypes.c_float(0.1), 0, 0, dummy, 1 << 30, None]
    # k_new without v_new
    assert lib.pa_decode_shared(dummy, dummy, dummy, None, *args[4:], 8, *rest) == pa.PA_ERR_INVALID
    # more sequences than one grouping takes are chunked, after the argument checks
    bad_dtype = rest[:8] + [7] + rest[9:]
    assert lib.pa_decode_shared(*args, 1025, *bad_dtype) == pa.PA_ERR_INVALID
    # 8-bit cache: format, scale arrays, then the same limits
    qargs = [dummy, dummy, dummy, dummy, dummy, dummy]
    qrest = [32, 8, 128, 16, 64, 4096, 1024, ctypes.c_float(0.1), 0]
    tail = [0, dummy, 1 << 30, None]
    assert lib.pa_decode_shared_quant(*qargs, 8, *qrest, 7, dummy, dummy, *tail) == pa.PA_ERR_INVALID
    assert lib.pa_decode_shared_quant(*qargs, 8, *qrest, pa.PA_KV_INT8, None, dummy, *tail) == pa.PA_ERR_INVALID
    qbad_dtype = qrest[:8] + [7]
    assert lib.pa_decode_shared_quant(*qargs, 1025, *qbad_dtype, pa.PA_KV_E4M3, dummy, dummy, *tail) == \
        pa.PA_ERR_INVALID


def _header_declarations():
    import re
    with open(pa.HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    decls = {}
    for m in re.finditer(r"PA_API\s+([\w\s\*]+?)\s*\b(pa_\w+)\s*\(([^)]*)\)\s*;", text):
        params = [x.strip() for x in m.group(3).split(",") if x.strip() and x.strip() != "void"]
        decls[m.group(2)] = (m.group(1).strip(), params)
    return decls


def _ctypes_kind(c_type: str):
    t = c_type.replace("const", "").strip()
    if "*" in t or t.startswith("pa_stream_t"):
        return "pointer"
    t = t.split()[:-1] if len(t.split()) > 1 else t.split()
    base = " ".join(t)
    return {"int": "int", "pa_dtype": "int", "pa_status": "int", "float": "float", "size_t": "u64",
            "unsigned long long": "u64", "unsigned int": "uint"}[base]


def test_binding_signatures_match_header():
    """Every function the header declares is set up in the binding with the
    same number and kinds of arguments (a mismatch would pass garbage)."""
    lib = pa.lib()
    # size_t and unsigned long long are both 64-bit unsigned here (one ctypes class)
    kinds = {ctypes.c_int: "int", ctypes.c_float: "float", ctypes.c_size_t: "u64",
             ctypes.c_ulonglong: "u64", ctypes.c_uint: "uint", ctypes.c_void_p: "pointer",
             ctypes.c_char_p: "pointer"}
    decls = _header_declarations()
    assert set(decls) == set(pa.header_functions())
    for name, (ret, params) in decls.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None, f"{name}: argtypes not set in the binding"
        assert len(fn.argtypes) == len(params), f"{name}: {len(fn.argtypes)} argtypes, header has {len(params)}"
        for i, (a, p) in enumerate(zip(fn.argtypes, params)):
            got = "pointer" if hasattr(a, "_type_") and a not in kinds else kinds.get(a)
            if a not in kinds and isinstance(a, type) and issubclass(a, ctypes._Pointer):
                got = "pointer"
            assert got == _ctypes_kind(p), f"{name} argument {i} ({p}): binding has {a}"
