"""The C-ABI libraries load, export every declared symbol, and reject bad
arguments on the host before touching the GPU (CPU only)."""
import ctypes
import math
import os
import re
import subprocess

import pytest

from exact_attention_152_b200 import binding, blocks_binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = {
    "attn.h": binding.LIB_PATH,
    "attn_blocks.h": blocks_binding.LIB_PATH,
}


def declared_functions(header_path):
    src = open(header_path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_]\w*\s*\**\s*([A-Za-z_]\w*)\s*\([^;{]*\)\s*;",
                       src, flags=re.M)
    return sorted(set(names))


def test_every_header_is_mapped():
    found = sorted(f for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h"))
    assert found == sorted(HEADERS), found


@pytest.mark.parametrize("header", sorted(HEADERS))
def test_library_exports_every_declared_symbol(header):
    lib_path = HEADERS[header]
    assert os.path.exists(lib_path), f"{lib_path} not built"
    names = declared_functions(os.path.join(ROOT, "include", header))
    assert names, "no declarations parsed"
    lib = ctypes.CDLL(lib_path)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # and they are real dynamic exports with C linkage (no C++ mangling)
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(names) <= exported, set(names) - exported


def test_attn_h_declares_the_contract():
    names = declared_functions(os.path.join(ROOT, "include", "attn.h"))
    for n in ("attn_fwd", "attn_fwd_config", "attn_fwd_gqa", "attn_status_sync", "attn_status_string",
              "attn_last_error", "attn_selftest_timeout"):
        assert n in names


def test_status_strings():
    for code in range(5):
        assert binding.attn_status_string(code)
    assert binding.attn_status_string(99) == "unknown status"


F = binding.attn_fwd
ALIGNED = 0x10000  # fake, never dereferenced: every case below fails validation first


@pytest.mark.parametrize("args,expect", [
    # negative sizes
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, -1, 1, 4, 4, 64, 0.1, 0), 1),
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, -4, 4, 64, 0.1, 0), 1),
    # non-finite scale
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 64, math.inf, 0), 1),
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 64, math.nan, 0), 1),
    # causal flag not 0/1
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 64, 0.1, 2), 1),
    # unsupported head dims
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 96, 0.1, 0), 2),
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 256, 0.1, 0), 2),
    # causal needs Nq == Nk
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 8, 64, 0.1, 1), 2),
    # null pointers with a non-empty problem
    ((None, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 64, 0.1, 0), 1),
    ((ALIGNED, ALIGNED, ALIGNED, None, None, 1, 1, 4, 4, 64, 0.1, 0), 1),
    # misaligned (q, o, lse)
    ((ALIGNED + 2, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 64, 0.1, 0), 1),
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16 + 8, None, 1, 1, 4, 4, 64, 0.1, 0), 1),
    ((ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, ALIGNED * 32 + 2, 1, 1, 4, 4, 64, 0.1, 0), 1),
    # o overlapping q / lse overlapping o
    ((ALIGNED, ALIGNED * 4, ALIGNED * 8, ALIGNED, None, 1, 1, 4, 4, 64, 0.1, 0), 1),
    ((ALIGNED, ALIGNED * 4, ALIGNED * 8, ALIGNED * 16, ALIGNED * 16 + 64, 1, 1, 4, 4, 64, 0.1, 0), 1),
    # empty problems are a no-op, even with null pointers
    ((None, None, None, None, None, 0, 4, 4, 4, 64, 0.1, 0), 0),
    ((None, None, None, None, None, 2, 4, 0, 4, 128, 0.1, 0), 0),
])
def test_host_validation(args, expect):
    assert F(*args, None) == expect


def test_gqa_validation():
    base = (ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1)
    # H % Hkv != 0, Hkv == 0, negative Hkv
    assert binding.attn_fwd_gqa(*base, 6, 4, 8, 8, 64, 0.1, 0, None) == 1
    assert binding.attn_fwd_gqa(*base, 6, 0, 8, 8, 64, 0.1, 0, None) == 1
    assert binding.attn_fwd_gqa(*base, 6, -2, 8, 8, 64, 0.1, 0, None) == 1
    # empty problem stays a no-op
    assert binding.attn_fwd_gqa(None, None, None, None, None, 0, 6, 2, 8, 8, 64, 0.1, 0, None) == 0
    # the other checks still apply
    assert binding.attn_fwd_gqa(*base, 6, 2, 8, 8, 96, 0.1, 0, None) == 2


def test_config_knob_validation():
    base = (ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 1, 4, 4, 64, 0.1, 0)
    assert binding.attn_fwd_config(*base, -1.0, 1, None, None) == 2
    assert binding.attn_fwd_config(*base, 65.0, 1, None, None) == 2
    assert binding.attn_fwd_config(*base, math.nan, 1, None, None) == 2
    assert binding.attn_fwd_config(*base, 8.0, 3, None, None) == 2
    assert binding.attn_fwd_config(*base, 8.0, -1, None, None) == 2
    # misaligned counter
    assert binding.attn_fwd_config(*base, 8.0, 1, ALIGNED * 64 + 4, None) == 1


def test_selftest_timeout_validation():
    assert binding.attn_selftest_timeout(0, None) == 1
    assert binding.attn_selftest_timeout(20_000_000, None) == 1


def test_blocks_validation():
    b = blocks_binding
    assert b.blocks_mma_ss(None, ALIGNED, ALIGNED, 64, None) == 1
    assert b.blocks_mma_ss(ALIGNED, ALIGNED, ALIGNED, 96, None) == 1
    assert b.blocks_mma_ts(ALIGNED + 4, ALIGNED, ALIGNED, 64, None) == 1
    assert b.blocks_swizzle_roundtrip(ALIGNED, ALIGNED, ALIGNED, 32, None) == 1
    assert b.blocks_exp2(None, None, None, -1, None) == 1
    assert b.blocks_exp2(None, None, None, 0, None) == 0
