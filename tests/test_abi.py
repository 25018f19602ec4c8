"""The C ABI library loads and exports every declared entry point; host-side argument
validation works without a GPU (no kernel is launched by these calls)."""
import ctypes
import os
import re

import pytest

import linear_attention_rnn_wkv_b200 as wkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wkv.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("wkv_forward", "wkv_decode_step", "token_shift_mix", "wkv_decode_step_fused",
                 "wkv_forward_workspace_size", "wkv_forward_status", "wkv_status_string"):
        assert must in names, names


def test_library_exports_every_declared_symbol():
    L = wkv.lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings():
    L = wkv.lib()
    for code, name in wkv.STATUS.items():
        assert L.wkv_status_string(code).decode() == name
    assert L.wkv_version() == 100


I64 = ctypes.c_int64
FAKE = 0x10000  # a 16-byte aligned, never dereferenced address


def _fwd(B, T, C, io=0, w=FAKE, u=FAKE, k=FAKE, v=FAKE, y=FAKE, st=None, ws=FAKE, nbytes=1 << 30, path=0, chunk=0):
    return wkv.lib().wkv_forward_ex(B, T, C, io, w, u, k, v, None, y, st, ws, nbytes, path, chunk, None)


def test_forward_validation_without_launch():
    assert _fwd(-1, 4, 4) == 1                   # negative size
    assert _fwd(1 << 40, 1 << 40, 4) == 1        # product overflows int64
    assert _fwd(1, 4, 4, io=7) == 3              # unknown dtype
    assert _fwd(1, 4, 4, path=9) == 3            # unknown path
    assert _fwd(1, 4, 4, chunk=5) == 3           # unsupported chunk
    assert _fwd(1, 4, 4, w=None) == 1            # null parameter
    assert _fwd(1, 4, 4, k=None) == 1            # null input
    assert _fwd(1, 4, 4, y=FAKE + 4) == 2        # misaligned output
    assert _fwd(1, 4, 4, k=FAKE + 8) == 2        # misaligned input
    assert _fwd(1, 4, 4, path=2, nbytes=16) == 1  # workspace too small for the chunked path
    assert _fwd(0, 4, 4) == 0 and _fwd(3, 4, 0) == 0  # empty calls are no-ops


def test_decode_and_shift_validation_without_launch():
    L = wkv.lib()
    assert L.wkv_decode_step(-2, 1, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert L.wkv_decode_step(2, 1, 4, FAKE, FAKE, None, FAKE, FAKE, FAKE, None) == 1
    assert L.wkv_decode_step(2, 1, 4, FAKE, FAKE, FAKE + 4, FAKE, FAKE, FAKE, None) == 2
    assert L.wkv_decode_step(0, 1, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 0
    assert L.wkv_decode_step_fused(2, 1, 4, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert L.token_shift_mix(1, 4, 4, FAKE, FAKE, FAKE + 4, FAKE, None) == 2
    assert L.token_shift_mix(1, 4, 4, None, FAKE, None, FAKE, None) == 1
    assert L.token_shift_mix(1, 0, 4, FAKE, FAKE, None, FAKE, None) == 0


def test_workspace_size_query():
    for (B, T, C) in [(1, 64, 64), (8, 1024, 768), (1, 16384, 4096), (3, 5, 7)]:
        n = wkv.lib().wkv_forward_workspace_size(B, T, C, 0)
        # header + a flag per tile + two 16-byte records per channel per tile; tiles span
        # 16 to 128 time steps and up to 128 channels (rounded up), so the size lies between
        lo = 64 + 2 * 16 * B * C * ((T + 127) // 128)
        hi = 64 + 16 + (4 + 2 * 32 * 128) * B * (C + 31) // 32 * ((T + 15) // 16)
        assert lo <= n <= hi, (n, lo, hi)
    assert wkv.lib().wkv_forward_workspace_size(0, 10, 10, 0) == 64


def test_binding_refuses_cpu_tensors():
    import torch
    k = torch.zeros(1, 4, 4)
    with pytest.raises(TypeError):
        wkv.wkv_forward(torch.ones(4), torch.zeros(4), k, k)
    with pytest.raises(TypeError):
        wkv.token_shift_mix(torch.ones(4), k)
    with pytest.raises(TypeError):
        wkv.wkv_backward(torch.ones(4), torch.zeros(4), k, k, k)
    with pytest.raises(TypeError):
        wkv.token_shift_mix3(torch.ones(4), torch.ones(4), torch.ones(4), k)
    k64 = torch.zeros(1, 4, 64)
    with pytest.raises(TypeError):
        wkv.eagle_forward(torch.ones(64), k64, k64, k64)
    with pytest.raises(TypeError):
        wkv.eagle_decode_step(torch.ones(1, 64), k64, k64, k64, torch.zeros(1, 4, 1, 64, 64))


def test_backward_validation_without_launch():
    """wkv_backward checks its arguments before touching the device (through the binding's
    argument types, so a wrong argument count fails here too)."""
    L = wkv.lib()

    def bwd(B, T, C, w=FAKE, k=FAKE, gk=FAKE, ws=FAKE, nbytes=1 << 30):
        return L.wkv_backward(B, T, C, w, FAKE, k, FAKE, FAKE, gk, FAKE, FAKE, FAKE, ws, nbytes, None)

    assert bwd(-1, 4, 4) == 1                    # negative size
    assert bwd(1, 4, 4, w=None) == 1             # null parameter
    assert bwd(1, 4, 4, k=None) == 1             # null input
    assert bwd(1, 4, 4, gk=FAKE + 4) == 2        # misaligned output
    assert bwd(1, 4, 4, nbytes=16) == 1          # workspace too small
    assert bwd(1 << 16, 1 << 20, 96) == 3        # more blocks than one launch's grid
    assert bwd(1 << 16, 1 << 20, 96, nbytes=16) == 3
    # a 64-byte header and 72 B per (b, group of 128 steps, c): the two published records
    assert L.wkv_backward_workspace_size(2, 3, 5) == 64 + 2 * 1 * 5 * 72
    assert L.wkv_backward_workspace_size(1, 130, 2) == 64 + 1 * 2 * 2 * 72
    assert L.wkv_backward_workspace_size(1, 128, 2) == 64 + 1 * 1 * 2 * 72
    assert L.wkv_backward_workspace_size(1, 129, 160) == 64 + 1 * 2 * 160 * 72


def test_gated_and_shift3_validation_without_launch():
    L = wkv.lib()
    gated = lambda r, y=FAKE: L.wkv_forward_gated(1, 4, 4, 0, FAKE, FAKE, FAKE, FAKE, r, None, y, None, FAKE,
                                                   1 << 30, 0, 0, None)
    assert gated(None) == 1                      # r is required
    assert gated(FAKE + 8) == 2                  # misaligned r
    shift3 = lambda x=FAKE, xr=FAKE: L.token_shift_mix3(1, 4, 4, FAKE, FAKE, FAKE, x, None, xr, FAKE, FAKE, None)
    assert shift3(x=None) == 1
    assert shift3(xr=FAKE + 4) == 2


def test_eagle_validation_without_launch():
    """eagle_forward / eagle_decode_step check their arguments before touching the device."""
    L = wkv.lib()

    def fwd(B, T, C, r=FAKE, y=FAKE, ws=FAKE, nbytes=1 << 30, state_in=None):
        return L.eagle_forward(B, T, C, FAKE, r, FAKE, FAKE, state_in, y, None, ws, nbytes, None)

    assert fwd(-1, 4, 64) == 1                   # negative size
    assert fwd(1, 4, 96) == 3                    # C not a multiple of the head size
    assert fwd(1, 4, 64, r=None) == 1            # null input
    assert fwd(1, 4, 64, y=FAKE + 4) == 2        # misaligned output
    assert fwd(1, 4, 64, state_in=FAKE + 8) == 2  # misaligned optional state
    assert fwd(1, 1000, 64, nbytes=16) == 1      # workspace too small (the three-launch form)
    assert fwd(70000, 1, 64) == 3                # batch above the grid's z limit
    assert fwd(0, 4, 64) == 0 and fwd(1, 4, 0) == 0  # empty calls
    # the one-launch form (24 or more sequence-heads, or at most 8 chunks) needs no scratch; the
    # three-launch form one 64 x 64 fp32 state per (sequence, head, 64-token chunk)
    assert L.eagle_forward_launches(2, 65, 128) == 1 and L.eagle_forward_workspace_size(2, 65, 128) == 0
    assert L.eagle_forward_launches(8, 1024, 768) == 1 and L.eagle_forward_workspace_size(8, 1024, 768) == 0
    assert L.eagle_forward_launches(1, 512, 64) == 1 and L.eagle_forward_workspace_size(1, 512, 64) == 0
    assert L.eagle_forward_launches(1, 513, 64) == 3
    assert L.eagle_forward_workspace_size(1, 1000, 64) == 16 * 64 * 64 * 4
    assert L.eagle_forward_workspace_size(2, 1000, 640) == 2 * 10 * 16 * 64 * 64 * 4
    assert L.eagle_forward_launches(3, 5000, 448) == 3 and L.eagle_forward_launches(4, 5000, 384) == 1
    assert L.eagle_forward_workspace_size(1, 4, 96) == 0 and L.eagle_forward_launches(1, 4, 96) == 0

    def dec(N, L_, C, state=FAKE, y=FAKE):
        return L.eagle_decode_step(N, L_, C, FAKE, FAKE, FAKE, FAKE, state, y, None)

    assert dec(2, 1, 100) == 3
    assert dec(2, 1, 64, state=None) == 1
    assert dec(2, 1, 64, y=FAKE + 4) == 2
    assert dec(0, 1, 64) == 0
