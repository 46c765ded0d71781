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
    for n in ("attn_fwd", "attn_fwd_config", "attn_fwd_gqa", "attn_fwd_window", "attn_fwd_varlen",
              "attn_fwd_fp8", "attn_fwd_colmask", "attn_colmask_workspace_size", "attn_bwd", "attn_bwd_window", "attn_bwd_varlen", "attn_bwd_colmask", "attn_bwd_colmask_workspace_size", "attn_bwd_noalloc", "attn_bwd_workspace_size", "attn_status_sync", "attn_status_string",
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


def test_window_validation():
    W = binding.attn_fwd_window
    base = (ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 4, 2, 8, 8, 64, 0.1)
    assert W(*base, -2, 0, None) == 1        # bounds below -1
    assert W(*base, 0, -5, None) == 1
    assert W(ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, 1, 4, 3, 8, 8, 64, 0.1, 3, 3, None) == 1
    assert W(*base[:10], 96, 0.1, 3, 3, None) == 2
    assert W(*base[:11], math.nan, 3, 3, None) == 1
    # empty problems are a no-op whatever the band
    assert W(None, None, None, None, None, 0, 4, 2, 8, 8, 64, 0.1, 3, 0, None) == 0


def test_colmask_validation():
    C = binding.attn_fwd_colmask
    P = (ALIGNED, ALIGNED * 2, ALIGNED * 3, ALIGNED * 16, None)
    sizes = (1, 4, 2, 8, 8, 64, 0.1, 0)            # B, H, Hkv, Nq, Nk, d, scale, causal
    M, WS = ALIGNED * 40, ALIGNED * 48
    need = binding.attn_colmask_workspace_size(1, 1, 8)
    # one key block: two int4 summaries (32 bytes, the minimum), then the CTA
    # plan's room: one int per mask row and 256-row block of up to 4 Nk query
    # rows, padded to 16 bytes
    assert need == 32 + 16
    assert binding.attn_colmask_workspace_size(2, 4, 129) == 2 * 4 * 2 * 32 + 2 * 4 * 3 * 4
    assert binding.attn_colmask_workspace_size(-1, 1, 8) == 0

    def call(ptrs=P, sz=sizes, mask=M, hm=1, ws=WS, ws_bytes=need):
        return C(*ptrs, *sz, mask, hm, ws, ws_bytes, None)
    assert call(sz=sizes[:7] + (2,)) == 1          # causal flag
    assert call(hm=3) == 1                         # Hm not in {1, H}
    assert call(mask=None) == 1
    assert call(ws=None) == 1
    assert call(mask=M + 4) == 1                   # misaligned mask
    assert call(ws=WS + 8) == 1                    # misaligned workspace
    assert call(ws_bytes=32 - 16) == 1             # workspace below the summaries
    assert call(ws=ALIGNED * 16) == 1              # workspace inside o
    assert call(ws=M) == 1                         # workspace over the mask
    assert call(mask=ALIGNED * 16) == 1            # mask inside o
    assert call(sz=(1, 4, 3) + sizes[3:]) == 1     # H % Hkv
    assert call(sz=sizes[:5] + (96,) + sizes[6:]) == 2
    # nothing to compute: a no-op even with null pointers
    assert C(None, None, None, None, None, 0, 4, 2, 8, 8, 64, 0.1, 0, None, 1, None, 0, None) == 0
    # more than 65536 key blocks of 128: unsupported (fake pointers far apart)
    T = 1 << 40
    nk = 65536 * 128 + 1
    big = binding.attn_colmask_workspace_size(1, 1, nk)
    assert C(T, 2 * T, 3 * T, 4 * T, None, 1, 1, 1, 8, nk, 64, 0.1, 0, 5 * T, 1, 6 * T, big, None) == 2


def test_varlen_validation():
    V = binding.attn_fwd_varlen
    P = (ALIGNED, ALIGNED, ALIGNED, ALIGNED * 16, None, ALIGNED * 64, ALIGNED * 65)
    ok_sizes = (2, 100, 150, 150, 4, 2, 64, 0.1, -1, 0)   # seqs, max_q, total_q, total_k, H, Hkv, d, ...
    def call(ptrs=P, sizes=ok_sizes):
        return V(*ptrs, *sizes, None)
    assert call(sizes=(-1,) + ok_sizes[1:]) == 1                      # negative num_seqs
    assert call(sizes=ok_sizes[:1] + (200,) + ok_sizes[2:]) == 1      # max_seqlen_q > total_q
    assert call(sizes=ok_sizes[:1] + (0,) + ok_sizes[2:]) == 1        # rows but no room for them
    assert call(sizes=ok_sizes[:5] + (3,) + ok_sizes[6:]) == 1        # H % Hkv != 0
    assert call(sizes=ok_sizes[:6] + (80,) + ok_sizes[7:]) == 2       # head dim
    assert call(sizes=ok_sizes[:7] + (math.inf,) + ok_sizes[8:]) == 1
    assert call(sizes=ok_sizes[:8] + (-3, 0)) == 1                    # band
    assert call(ptrs=P[:5] + (None,) + P[6:]) == 1                    # null offsets
    assert call(ptrs=P[:5] + (ALIGNED * 64 + 2,) + P[6:]) == 1        # misaligned offsets
    assert call(ptrs=(ALIGNED + 8,) + P[1:]) == 1                     # misaligned q
    assert call(ptrs=P[:3] + (ALIGNED,) + P[4:]) == 1                 # o overlaps q
    assert call(ptrs=P[:5] + (ALIGNED * 16,) + P[6:]) == 1            # offsets inside o
    # nothing to compute: a no-op even with null pointers
    assert V(None, None, None, None, None, None, None, 0, 0, 0, 0, 4, 2, 64, 0.1, -1, 0, None) == 0
    assert V(None, None, None, None, None, None, None, 3, 0, 0, 0, 4, 2, 64, 0.1, -1, 0, None) == 0


def test_fp8_validation():
    F8 = binding.attn_fwd_fp8
    P = (ALIGNED, ALIGNED * 2, ALIGNED * 3, ALIGNED * 16, None)
    assert F8(*P, 1, 2, 2, 64, 64, 64, 0.1, 1.0, 1.0, 1.0, 0, None) == 2      # d must be 128
    assert F8(*P, 1, 2, 2, 64, 32, 128, 0.1, 1.0, 1.0, 1.0, 1, None) == 2     # causal Nq != Nk
    assert F8(*P, 1, 2, 2, 64, 64, 128, 0.1, math.nan, 1.0, 1.0, 0, None) == 1
    assert F8(*P, 1, 2, 2, 64, 64, 128, 0.1, 1.0, 1.0, math.inf, 0, None) == 1
    assert F8(*P, 1, 2, 2, 64, 64, 128, 1e30, 1e30, 1.0, 1.0, 0, None) == 1  # scale product overflows
    assert F8(*P, 1, 3, 2, 64, 64, 128, 0.1, 1.0, 1.0, 1.0, 0, None) == 1     # H % Hkv
    assert F8(ALIGNED + 1, *P[1:], 1, 2, 2, 64, 64, 128, 0.1, 1.0, 1.0, 1.0, 0, None) == 1
    assert F8(None, None, None, None, None, 0, 2, 2, 64, 64, 128, 0.1, 1.0, 1.0, 1.0, 0, None) == 0


def test_bwd_validation():
    Bw = binding.attn_bwd
    A = ALIGNED
    ptrs = (A, A * 2, A * 3, A * 4, A * 5, A * 6, A * 7, A * 8, A * 9, A * 16)
    need = binding.attn_bwd_workspace_size(1, 2, 64, 64)
    assert need == 512 + 1 * 2 * 64 * 64 * 4   # row sums (256-aligned) + fp32 dQ
    assert binding.attn_bwd_workspace_size(1, 2, 64, 96) == 0
    sizes = (1, 2, 2, 64, 64, 64, 0.1, 0)
    assert Bw(*ptrs, need - 1, *sizes, None) == 1                # workspace too small
    assert Bw(*ptrs[:9], None, need, *sizes, None) == 1          # no workspace
    assert Bw(*ptrs[:9], A * 16 + 16, need, *sizes, None) == 1   # workspace misaligned (256)
    assert Bw(*ptrs, need, 1, 2, 2, 64, 64, 80, 0.1, 0, None) == 2
    assert Bw(*ptrs, need, 1, 2, 2, 64, 32, 64, 0.1, 1, None) == 2   # causal Nq != Nk
    assert Bw(*ptrs, need, 1, 3, 2, 64, 64, 64, 0.1, 0, None) == 1   # H % Hkv
    assert Bw(*ptrs, need, 1, 2, 2, 64, 64, 64, math.inf, 0, None) == 1
    assert Bw(*ptrs[:6], A, *ptrs[7:], need, *sizes, None) == 1   # dq overlaps q
    assert Bw(*ptrs[:9], A * 9, need, *sizes, None) == 1         # workspace overlaps dv
    assert Bw(*(None,) * 10, 0, 0, 2, 2, 64, 64, 64, 0.1, 0, None) == 0   # empty batch
    BW = binding.attn_bwd_window
    assert BW(*ptrs, need, 1, 2, 2, 64, 64, 64, 0.1, -2, 0, None) == 1    # band below -1
    assert BW(*ptrs, need, 1, 2, 2, 64, 64, 64, 0.1, 0, -3, None) == 1
    assert BW(*ptrs, need - 1, 1, 2, 2, 64, 64, 64, 0.1, 8, 0, None) == 1  # workspace too small


def test_bwd_colmask_validation():
    BC = binding.attn_bwd_colmask
    A = ALIGNED
    ptrs = (A, A * 2, A * 3, A * 4, A * 5, A * 6, A * 7, A * 8, A * 9, A * 16)
    base = binding.attn_bwd_workspace_size(1, 2, 64, 64)
    need = binding.attn_bwd_colmask_workspace_size(1, 2, 64, 64, 1, 64)
    minimum = (base + 255) // 256 * 256 + 32           # + one key block's two int4 summaries
    assert need == minimum + 16                        # + the CTA plan: 2 ints, padded to 16 bytes
    assert binding.attn_bwd_colmask_workspace_size(1, 2, 64, 96, 1, 64) == 0
    M = A * 40
    sizes = (1, 2, 2, 64, 64, 64, 0.1, 0)

    def call(ws=need, mask=M, hm=1, sz=sizes, p=ptrs):
        return BC(*p, ws, *sz, mask, hm, None)
    assert call(ws=minimum - 1) == 1                   # workspace too small
    assert call(ws=base) == 1                          # room for attn_bwd only
    assert call(mask=None) == 1
    assert call(mask=M + 4) == 1                       # misaligned mask
    assert call(hm=3) == 1                             # Hm not in {1, H}
    assert call(mask=A * 7) == 1                       # mask inside dq
    assert call(sz=sizes[:7] + (2,)) == 1              # causal flag
    assert call(sz=sizes[:5] + (80,) + sizes[6:]) == 2


def test_bwd_varlen_validation():
    BV = binding.attn_bwd_varlen
    A = ALIGNED
    ptrs = (A, A * 2, A * 3, A * 4, A * 5, A * 6, A * 7, A * 8, A * 9, A * 16)
    need = binding.attn_bwd_workspace_size(1, 2, 150, 64)
    cu = (A * 64, A * 65)
    sizes = (2, 100, 150, 150, 2, 2, 64, 0.1, -1, 0)  # seqs, max_k, total_q, total_k, H, Hkv, d, ...

    def call(p=ptrs, ws=need, c=cu, sz=sizes):
        return BV(*p, ws, *c, *sz, None)
    assert call(ws=need - 1) == 1                                   # workspace too small
    assert call(c=(None, A * 65)) == 1                              # null offsets
    assert call(c=(A * 64 + 2, A * 65)) == 1                        # misaligned offsets
    assert call(sz=(2, 200) + sizes[2:]) == 1                       # max_seqlen_k > total_k
    assert call(sz=(2, 0) + sizes[2:]) == 1                         # keys but max_seqlen_k 0
    assert call(sz=sizes[:5] + (3,) + sizes[6:]) == 1               # H % Hkv
    assert call(sz=sizes[:6] + (96,) + sizes[7:]) == 2              # head dim
    assert call(sz=sizes[:8] + (-2, 0)) == 1                        # band
    assert call(p=ptrs[:6] + (A,) + ptrs[7:]) == 1                  # dq overlaps q
    assert call(c=(A * 7, A * 65)) == 1                             # offsets inside dq
    assert BV(*(None,) * 10, 0, None, None, 0, 0, 0, 0, 2, 2, 64, 0.1, -1, 0, None) == 0


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
