"""The C-ABI library loads on a machine without a GPU and exports every entry point that
include/lora_sgmv.h declares; host-only calls behave as documented.  No compute call is made."""
import ctypes
import os
import re

import pytest

import heterogeneous_adapters_sgmv_b200 as L
from heterogeneous_adapters_sgmv_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "lora_sgmv.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lora_\w+)\s*\(", txt)))


def test_library_builds_and_exports_every_declared_symbol():
    path = B.build()
    lib = ctypes.CDLL(path)
    names = declared_functions()
    assert len(names) >= 13
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(L.EXPORTS) == names


def test_host_only_calls():
    L._load()
    assert L.status_string(L.LORA_ERR_WORKSPACE).startswith("workspace")
    assert L.status_string(12345) == "unknown status"
    lib = L._load()
    assert lib.lora_table_info(None, None, None, None, None, None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_workspace_bytes(None, 5) == 256
    assert lib.lora_table_destroy(None) == L.LORA_OK
    # grouped call: argument checks that need no table
    arr = (ctypes.c_void_p * 5)()
    i64 = (ctypes.c_int64 * 5)()
    i32 = (ctypes.c_int32 * 5)()
    seg = L.lora_segments()
    for P in (0, 5, -1):
        assert lib.lora_sgmv_grouped(arr, P, ctypes.byref(seg), arr, i64, arr, i64, i32, None, 0,
                                     None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_sgmv_grouped(None, 1, ctypes.byref(seg), arr, i64, arr, i64, i32, None, 0,
                                 None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_sgmv_grouped(arr, 1, ctypes.byref(seg), arr, i64, arr, i64, i32, None, 0,
                                 None) == L.LORA_ERR_INVALID_ARG   # null segment pointers / table
    old = L.lora_get_option("split")
    L.lora_set_option("split", 1)
    assert L.lora_get_option("split") == 1
    L.lora_set_option("split", old)
    try:
        L.lora_set_option("no_such_knob", 1)
        raise AssertionError("unknown option accepted")
    except L.LoraError as e:
        assert e.code == L.LORA_ERR_INVALID_ARG
    assert lib.lora_table_create(None, 1, 8, 8, 1, None, None, None, None, None) == L.LORA_ERR_INVALID_ARG


def test_header_constants_match_binding():
    txt = open(os.path.join(ROOT, "include", "lora_sgmv.h")).read()
    for name in ("LORA_F32", "LORA_BF16", "LORA_OK", "LORA_ERR_INVALID_ARG", "LORA_ERR_UNSUPPORTED",
                 "LORA_ERR_WORKSPACE", "LORA_ERR_CUDA", "LORA_ERR_TIMEOUT", "LORA_ERR_DEVICE_STATUS",
                 "LORA_STATUS_BAD_ID", "LORA_STATUS_TIMEOUT", "LORA_STATUS_BAD_SEGMENT", "LORA_MAX_RANK",
                 "LORA_MAX_SEGMENT_TOKENS", "LORA_NOALLOC_SCRATCH_FLOATS", "LORA_MAX_GROUP",
                 "LORA_SIGMA_NONE", "LORA_SIGMA_FULL", "LORA_SIGMA_DIAG", "LORA_MAX_MERGE",
                 "LORA_KERNEL_KINDS"):
        m = re.search(r"#define %s \(?(-?\d+)u?\)?" % name, txt)
        assert m, name
        assert int(m.group(1)) == getattr(L, name), name


def test_product_path_does_not_use_the_oracle():
    """The package neither imports nor names the oracle: no CPU fallback exists."""
    pkg = os.path.join(ROOT, "heterogeneous_adapters_sgmv_b200")
    for dirpath, _d, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read().lower()
                assert "oracle" not in src, f


def test_every_documented_option_round_trips():
    """Each runtime option the header documents can be set and read back (host only), and an
    unknown key is rejected."""
    txt = open(os.path.join(ROOT, "include", "lora_sgmv.h")).read()
    block = txt[txt.index("Runtime knobs"):txt.index("int lora_set_option")]
    keys = re.findall(r'"([a-z_]+)"', block)
    assert {"pdl", "decode_stages", "decode_ctas_per_sm", "decode_cluster", "decode_max_clusters",
            "prefill_ksplit", "prefill_min_seg_len", "split"} <= set(keys)
    for key in keys:
        old = L.lora_get_option(key)
        try:
            L.lora_set_option(key, old + 3)
            assert L.lora_get_option(key) == old + 3
        finally:
            L.lora_set_option(key, old)
        assert L.lora_get_option(key) == old
    with pytest.raises(L.LoraError):
        L.lora_set_option("no_such_option", 1)


def test_launch_counters_name_every_kernel():
    """The launch counters cover each __global__ kernel of the library by name, start at a
    count of zero or more, and reject kinds outside the range (host only)."""
    lib = L._load()
    names = [lib.lora_kernel_name(k).decode() for k in range(L.LORA_KERNEL_KINDS)]
    assert lib.lora_kernel_name(-1) is None and lib.lora_kernel_name(L.LORA_KERNEL_KINDS) is None
    assert lib.lora_kernel_launches(-1) == -1 and lib.lora_kernel_launches(L.LORA_KERNEL_KINDS) == -1
    src = ""
    csrc = os.path.join(ROOT, "heterogeneous_adapters_sgmv_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith(".cu"):
            src += open(os.path.join(csrc, f)).read()
    kernels = set(re.findall(r"__global__ void(?: __launch_bounds__\([^)]*\))?\s+(\w+)\(", src))
    assert kernels == set(names), (kernels, names)
    counts = L.kernel_launches()
    assert set(counts) == set(names) and all(v >= 0 for v in counts.values())


def test_merged_and_sigma_host_checks():
    """Argument checks of the next-row entry points that need no device."""
    lib = L._load()
    assert lib.lora_table_set_sigma(None, L.LORA_SIGMA_FULL, None, None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_bgmv_merged(None, None, None, 4, 2, None, 0, None, 0, 0, None, 0, None) == \
        L.LORA_ERR_INVALID_ARG
