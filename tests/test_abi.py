"""The C ABI boundary, checked without a GPU: the library loads, exports every
symbol include/fa.h declares, and rejects invalid arguments on the host before
any CUDA call (so nothing is launched and no output is touched)."""
import ctypes
import os
import re

import pytest

import exact_io_aware_44_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "fa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("fa_fwd", "fa_fwd_f32", "fa_bwd", "fa_bwd_workspace_bytes", "fa_get_status", "fa_error_string"):
        assert s in syms


def test_every_declared_symbol_is_exported():
    so = ctypes.CDLL(fa.LIB_PATH)
    for s in declared_symbols():
        assert hasattr(so, s), s
        assert s in fa.SIGNATURES, f"binding lacks {s}"


def test_library_has_sm100a_code_only_and_static_runtime():
    # the shared object must not need libcudart.so at load time
    import subprocess
    out = subprocess.run(["ldd", fa.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart.so" not in out
    assert "libcuda.so" not in out


def test_version_and_error_strings():
    assert fa.lib.fa_version() >= 100
    for code in list(fa.STATUS) + [12345]:
        assert fa.lib.fa_error_string(code)


def _fwd(d=64, B=1, Hq=2, Hkv=1, N=128, causal=1, scale=0.125, ptr=0x1000, f32=False):
    return fa.fwd_raw(ptr, ptr, ptr, ptr, ptr, B, Hq, Hkv, N, d, causal, scale, 0, f32=f32)


def test_invalid_arguments_rejected_on_host():
    assert _fwd(d=96) == -2                       # unsupported head dim
    assert _fwd(d=64, Hq=3, Hkv=2) == -1          # Hq not a multiple of Hkv
    assert _fwd(B=0) == -1
    assert _fwd(scale=0.0) == -1
    assert _fwd(scale=float("nan")) == -1
    assert _fwd(scale=float("inf")) == -1
    assert _fwd(N=-1) == -1
    assert _fwd(ptr=0x1008) == -3                 # not 16-byte aligned
    assert _fwd(ptr=0) == -1                      # null pointers
    assert _fwd(N=0, ptr=0) == 0                  # empty problem: nothing to do
    assert _fwd(d=102, f32=True) == -2            # fp32 path: d % 4 != 0
    assert _fwd(d=132, f32=True) == -2            # fp32 path: d > 128
    assert _fwd(B=1 << 12, Hq=1 << 10, Hkv=1, N=1 << 10) == -2   # B*Hq*N >= 2^31


def _fwd8(d=128, N=128, ds=(0.01, 0.02, 0.03), ptr=0x1000, scale=0.088):
    return fa.fwd_fp8_raw(ptr, ptr, ptr, *ds, ptr, ptr, 1, 2, 1, N, d, 1, scale, 0)


def test_fp8_forward_rejects_bad_arguments_on_host():
    assert _fwd8(d=64) == -2                      # E4M3 path: d = 128 only
    assert _fwd8(ds=(0.0, 0.02, 0.03)) == -1      # descales must be positive and finite
    assert _fwd8(ds=(0.01, -1.0, 0.03)) == -1
    assert _fwd8(ds=(0.01, 0.02, float("inf"))) == -1
    assert _fwd8(ds=(0.01, float("nan"), 0.03)) == -1
    assert _fwd8(ds=(1e30, 1e30, 1.0)) == -1      # scale * descale_q * descale_k overflows
    assert _fwd8(scale=0.0) == -1
    assert _fwd8(ptr=0x1004) == -3
    assert _fwd8(N=0, ptr=0) == 0


def _dec(B=1, Hq=8, Hkv=1, Nq=1, Nk=1000, d=128, causal=1, scale=0.088, splits=0, ptr=0x1000, ws=0x1000):
    return fa.decode_raw(ptr, ptr, ptr, ptr, ptr, ws, B, Hq, Hkv, Nq, Nk, d, causal, scale, splits, 0)


def test_decode_rejects_bad_arguments_on_host():
    assert _dec(d=256) == -2                       # d = 64 or 128
    assert _dec(d=64, ptr=0x1008) == -3            # d = 64: accepted up to the pointer check
    assert _dec(Hq=64, Hkv=1, ptr=0x1008) == -3    # 64 query rows per group: accepted up to the pointer check
    assert _dec(Hq=8, Nq=5, ws=0x1010) == -3       # 40 rows: row blocks, past the size checks
    assert _dec(Hq=16, Nq=3000, Nk=3000, ptr=0x1008) == -3   # 48000 rows: 375 row blocks
    assert _dec(Nq=5, Nk=4) == -1                  # causal needs Nq <= Nk
    assert _dec(Nk=0) == -1
    assert _dec(Hq=6, Hkv=4) == -1
    assert _dec(scale=float("nan")) == -1
    assert _dec(ws=0x1010) == -3                   # workspace 256-byte aligned
    assert _dec(ptr=0x1008) == -3
    assert _dec(ws=0) == -1


def _decode_split(B, Hq, Hkv, Nq, Nk, splits, d=128):
    """The work split restated: a group of up to 32 query rows is one unit, a larger
    one is ceil(rows / 128) row blocks of 128; all units' 128-key chunks end to end,
    cut into n_ctas equal slices (one per SM of a 148-SM part, or units * num_splits;
    never more than the chunks); one workspace slot per (unit, CTA) pair that can
    meet, i.e. units + n_ctas - 1, each of slot_rows rows. At d = 64 a group of at most
    64 rows keeps two partial rows per query row (one per half of every key chunk), in
    slots of 128 rows."""
    rows = Hq // Hkv * Nq
    n_rb = 1 if rows <= 32 else -(-rows // 128)
    slot_rows = 128 if (d == 64 and rows <= 64) else rows if n_rb == 1 else 128
    n_chunks = -(-Nk // 128)
    units = B * Hkv * n_rb
    n_ctas = min(units * splits if splits > 0 else 148, units * n_chunks)
    return units + n_ctas - 1, slot_rows, units


def test_decode_workspace_and_split_rule():
    """Per slot: fp32 partial O (256-byte padded as a whole) and fp32 partial LSE per
    query row of a slot."""
    d = 128
    for (B, Hq, Hkv, Nq) in ((4, 32, 8, 1), (16, 32, 8, 1), (16, 32, 4, 4), (1, 8, 1, 3), (64, 16, 8, 1),
                             (16, 64, 1, 1), (2, 8, 1, 5), (16, 32, 2, 8), (1, 16, 1, 17), (3, 4, 1, 100)):
        for Nk, splits in ((128, 1), (4096, 4), (4096, 7), (100000, 0), (32768, 0), (777, 0), (1, 0), (200, 0)):
            if Nq > Nk:
                continue
            ws = fa.decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, splits)
            slots, slot_rows, units = _decode_split(B, Hq, Hkv, Nq, Nk, splits)
            pad = lambda x: (x + 255) // 256 * 256
            assert ws == pad(slots * slot_rows * d * 4) + slots * slot_rows * 4, (B, Hq, Hkv, Nq, Nk, splits, ws)
    assert fa.decode_workspace_bytes(1, 8, 1, 1, 1000, 256, 0) == 0
    # d = 64: the same split rule, d = 64 floats per partial row; up to 64 rows a group, two
    # partial rows per query row
    pad = lambda x: (x + 255) // 256 * 256
    for (B, Hq, Hkv, Nq) in ((2, 8, 2, 3), (16, 64, 8, 8), (2, 8, 1, 9), (1, 16, 1, 40)):
        slots, slot_rows, _ = _decode_split(B, Hq, Hkv, Nq, 1000, 0, d=64)
        assert slot_rows == (128 if Hq // Hkv * Nq <= 64 else Hq // Hkv * Nq if Hq // Hkv * Nq <= 128 else 128)
        assert fa.decode_workspace_bytes(B, Hq, Hkv, Nq, 1000, 64, 0) == \
            pad(slots * slot_rows * 64 * 4) + slots * slot_rows * 4, (B, Hq, Hkv, Nq)


def test_bwd_rejects_bad_arguments_on_host():
    p = 0x1000
    r = fa.bwd_raw(p, p, p, p, p, p, p, p, p, p + 16, 1, 2, 1, 128, 64, 1, 0.125, 0)
    assert r == -3                                # workspace must be 256-byte aligned
    r = fa.bwd_raw(p, p, p, p, p, p, p, p, p, 0, 1, 2, 1, 128, 64, 1, 0.125, 0)
    assert r == -1
    r = fa.bwd_raw(p, p, p, p, p, p, p, p, p, p, 1, 2, 1, 128, 80, 1, 0.125, 0)
    assert r == -2


def test_workspace_is_linear_in_n():
    """The backward's scratch is O(N): D (fp32 per row) and the fp32 dQ accumulator."""
    B, Hq, Hkv, d = 2, 8, 2, 128
    sizes = [fa.workspace_bytes(B, Hq, Hkv, N, d) for N in (1024, 2048, 4096, 8192)]
    per_row = B * Hq * (d + 1) * 4
    for N, s in zip((1024, 2048, 4096, 8192), sizes):
        assert per_row * N <= s <= per_row * N + 256
    assert fa.workspace_bytes(0, 1, 1, 8, 64) == 0


def test_no_device_is_reported_without_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd() == -6
    assert fa.lib.fa_get_status(None) == -6


def test_progress_record_rejects_bad_arguments_on_host():
    import ctypes
    buf = (ctypes.c_uint * 4)()
    assert fa.lib.fa_get_progress(None, 4, None) == -1
    assert fa.lib.fa_get_progress(ctypes.cast(buf, ctypes.c_void_p), -1, None) == -1
