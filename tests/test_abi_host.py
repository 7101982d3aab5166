"""The C-ABI library loads, exports every symbol the header declares, and rejects invalid calls on
the host before any launch (CPU only: these paths make no CUDA call)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import exact_attention_160_b200 as ea

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_b200.h")


@pytest.fixture(scope="module")
def lib():
    from exact_attention_160_b200 import build
    build.build()
    return ea.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert set(names) == set(ea.EXPORTS), names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"


FAKE = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: validation rejects first


def fwd(lib, B=1, Hq=2, Hkv=2, Sq=8, Skv=8, D=64, scale=0.125, causal=0, dtype=0, ptr=FAKE):
    return lib.attn_fwd(ptr, ptr, ptr, ptr, None, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, None)


def test_fwd_validation(lib):
    assert fwd(lib, B=0) == 1
    assert fwd(lib, Sq=-1) == 1
    assert fwd(lib, Skv=0) == 3                   # empty KV (flash_decode.rs EmptyKv)
    assert fwd(lib, Hq=3, Hkv=2) == 2             # Hq not a multiple of Hkv
    assert fwd(lib, D=96) == 4                    # head dims other than 64/128
    assert fwd(lib, scale=0.0) == 1
    assert fwd(lib, scale=float("nan")) == 1
    assert fwd(lib, causal=2) == 1
    assert fwd(lib, dtype=7) == 1
    assert fwd(lib, dtype=2, D=96) == 4
    assert fwd(lib, ptr=None) == 1
    assert fwd(lib, ptr=ctypes.c_void_p((1 << 20) + 2)) == 1   # misaligned


def test_fwd_ex_validation(lib):
    P = FAKE
    need = lib.attn_fwd_ex_workspace_size(1, 2, 2, 8, 8, 64, 0, 10000.0, 0)
    assert need > 0
    assert lib.attn_fwd_ex_workspace_size(1, 2, 2, 8, 8, 64, 0, 0.0, 0) == 0
    # workspace missing / too small
    assert lib.attn_fwd_ex(P, P, P, P, None, 1, 2, 2, 8, 8, 64, 0.1, 1, 0, 10000.0, 0, None, 0, None) == 5
    assert lib.attn_fwd_ex(P, P, P, P, None, 1, 2, 2, 8, 8, 64, 0.1, 1, 0, 10000.0, 0, P, need - 1, None) == 5
    assert lib.attn_fwd_ex(P, P, P, P, None, 1, 2, 2, 8, 8, 64, 0.1, 1, 0, 10000.0, -1, P, need, None) == 1


def test_fwd_masked_validation(lib):
    """attn_fwd_masked rejects a missing or misaligned mask and negative strides, and applies the
    forward's own checks, before any launch."""
    P = FAKE

    def call(mask=P, bs=0, hs=0, B=1, Hq=2, Hkv=2):
        return lib.attn_fwd_masked(P, P, P, mask, bs, hs, P, None, B, Hq, Hkv, 8, 8, 64, 0.125, 0, 0, 0.0, 0,
                                   None, 0, None)
    assert call(mask=None) == 1
    assert call(mask=ctypes.c_void_p((1 << 20) + 2)) == 1     # not 4-byte aligned
    assert call(bs=-1) == 1
    assert call(hs=-64) == 1
    assert call(B=0) == 1
    assert call(Hq=3, Hkv=2) == 2


def test_fwd_key_split_sizing(lib):
    """Key splits: n = min(148 // tiles, ceil(Skv/128) // 2, 16) for bf16 problems of <= 74 query
    tiles, taken when they spare the longest chunk >= 8 key tiles; their partials (splits x rows x
    (D + 1) floats) follow the RoPE part of the workspace."""
    assert lib.attn_fwd_kv_splits(1, 6, 1500, 1500, 0) == 1      # 72 tiles, 12 key tiles: spares 6
    assert lib.attn_fwd_kv_splits(1, 2, 1500, 2100, 0) == 6      # 24 tiles, 17 key tiles: spares 14
    assert lib.attn_fwd_kv_splits(1, 8, 128, 4096, 0) == 16      # 8 tiles, 32 key tiles
    assert lib.attn_fwd_kv_splits(1, 2, 300, 2100, 2) == 8       # bf16 in, fp32 out
    assert lib.attn_fwd_kv_splits(1, 2, 300, 1000, 2) == 1       # 8 key tiles in 4 chunks: spares 6
    assert lib.attn_fwd_kv_splits(4, 8, 2048, 2048, 0) == 1      # 512 tiles
    assert lib.attn_fwd_kv_splits(1, 2, 300, 300, 0) == 1        # 3 key tiles
    assert lib.attn_fwd_kv_splits(1, 8, 128, 4096, 1) == 1       # fp32 path
    assert lib.attn_fwd_kv_splits(0, 8, 128, 4096, 0) == 1
    rows = 128 * 8
    part = -(-16 * rows * 64 * 4 // 256) * 256 + -(-16 * rows * 4 // 256) * 256
    assert lib.attn_fwd_ex_workspace_size(1, 8, 2, 128, 4096, 64, 0, 0.0, 0) == part
    assert lib.attn_fwd_ex_workspace_size(1, 6, 6, 1500, 1500, 64, 0, 0.0, 0) == 0   # unsplit, no RoPE
    # RoPE part: cos/sin table (4096 positions x 32 pairs x 8 B), then K hi and lo (bf16)
    rope = 4096 * 32 * 8 + 2 * (4096 * 2 * 64 * 2)
    assert lib.attn_fwd_ex_workspace_size(1, 8, 2, 128, 4096, 64, 0, 10000.0, 0) == rope + part
    # a non-NULL workspace below the size is refused before any launch
    P = FAKE
    assert lib.attn_fwd_ex(P, P, P, P, None, 1, 8, 2, 128, 4096, 64, 0.125, 0, 0, 0.0, 0, P, part - 1,
                           None) == 5


def test_key_split_count_follows_its_documented_rule(lib):
    """attn_fwd_kv_splits against the header's formula over a grid of sizes."""
    def rule(B, Hq, Sq, Skv, dtype):
        tiles = -(-Sq // 128) * B * Hq
        if dtype == 1 or tiles > 74:
            return 1
        nkv = -(-Skv // 128)
        n = min(148 // tiles, nkv // 2, 16)
        if n < 2:
            return 1
        return n if nkv - (-(-nkv // n)) >= 8 else 1
    for B in (1, 2, 3):
        for Hq in (1, 2, 6, 8, 32):
            for Sq in (1, 127, 128, 129, 700, 1500, 4096):
                for Skv in (1, 255, 256, 511, 512, 1500, 4096, 65536):
                    for dtype in (0, 1, 2):
                        assert lib.attn_fwd_kv_splits(B, Hq, Sq, Skv, dtype) == rule(B, Hq, Sq, Skv, dtype), \
                            (B, Hq, Sq, Skv, dtype)


def test_missing_library_fails_loudly(tmp_path):
    """No fallback: a binding whose library is absent raises instead of computing anything."""
    code = f"import exact_attention_160_b200 as ea; ea.load_library({str(tmp_path / 'absent.so')!r})"
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode != 0 and "not found" in r.stderr


def test_decode_validation(lib):
    P = FAKE
    need = lib.attn_decode_workspace_size(2, 8, 64, 4)
    assert need >= 2 * 8 * 4 * 64 * 4 + 2 * 8 * 4 * 4
    call = lambda **kw: lib.attn_decode(P, P, P, P, P, None, kw.get("B", 2), kw.get("Hq", 8), kw.get("Hkv", 2),
                                        kw.get("Smax", 100), kw.get("D", 64), kw.get("scale", 0.125),
                                        kw.get("ns", 4), kw.get("ws", P), kw.get("wsb", need),
                                        kw.get("dtype", 0), None)
    assert call(Smax=0) == 3
    assert call(Hq=6, Hkv=4) == 2
    assert call(ns=0) == 1
    assert call(wsb=need - 1) == 5
    assert call(ws=None) == 5
    assert call(dtype=1) == 4
    assert call(D=80) == 4


def test_rope_validation(lib):
    P = FAKE
    assert lib.rope_apply(P, P, 4, 2, 7, 10000.0, 0, None) == 2      # odd head dim
    assert lib.rope_apply(P, P, 0, 2, 8, 10000.0, 0, None) == 1
    assert lib.rope_apply(P, P, 4, 2, 8, -1.0, 0, None) == 1


def test_status_strings(lib):
    for s in range(8):
        assert lib.attn_status_string(s).decode() == ea.STATUS[s]
