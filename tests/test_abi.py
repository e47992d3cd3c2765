"""C-ABI checks that need no GPU: the library loads, exports what the header
declares, and rejects bad arguments on the host before touching CUDA."""

import ctypes

import pytest

import exact_attention_135_b200 as ea
from exact_attention_135_b200 import build as ea_build


@pytest.fixture(scope="module")
def lib():
    ea_build.build()
    return ea.library()


def test_header_symbols_exported(lib):
    names = ea.exported_symbols()
    assert {"attn_fwd", "attn_decode_paged", "attn_decode_paged_workspace_size", "attn_status_string",
            "attn_read_device_status", "attn_abi_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in the header but not exported"


def test_status_strings(lib):
    assert lib.attn_abi_version() == 1
    for code, name in ea.STATUS.items():
        assert lib.attn_status_string(code).decode() == name
    assert lib.attn_status_string(99).decode() == "ATTN_ERR_UNKNOWN"


A = 0x10000   # fake 16-byte aligned addresses: never dereferenced on the error paths below


def _fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, Hq=2, Hkv=2, Nq=128, Nk=128, D=64, Dv=64, causal=0, scale=0.125):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, Dv, causal, scale, None)


def test_fwd_rejects_bad_arguments(lib):
    assert _fwd(lib, q=None) == 1
    assert _fwd(lib, lse=None) == 1
    assert _fwd(lib, k=A + 8) == 1            # misaligned
    assert _fwd(lib, lse=A + 2) == 1
    assert _fwd(lib, Hq=3, Hkv=2) == 1        # Hq % Hkv
    assert _fwd(lib, B=0) == 1
    assert _fwd(lib, Nq=-1) == 1
    assert _fwd(lib, scale=0.0) == 1
    assert _fwd(lib, scale=-1.0) == 1
    assert _fwd(lib, scale=float("nan")) == 1
    assert _fwd(lib, scale=float("inf")) == 1
    assert _fwd(lib, B=70000) == 1


def test_fwd_unsupported_shapes(lib):
    assert _fwd(lib, D=96, Dv=96) == 2
    assert _fwd(lib, D=128, Dv=64) == 2
    assert _fwd(lib, D=32, Dv=32) == 2


def test_fwd_empty_query_is_noop(lib):
    assert _fwd(lib, Nq=0) == 0


def test_fwd_no_keys_accepts_null_kv_and_empty_query(lib):
    # Nq == 0: nothing to do, no CUDA call, even with null K/V
    assert _fwd(lib, k=None, v=None, Nq=0, Nk=0) == 0
    # Nk > 0 with null K is an argument error
    assert _fwd(lib, k=None, Nk=5) == 1


def test_selftest_rejects_bad_limits_on_host(lib):
    assert lib.attn_selftest_wait_timeout(0, None) == 1
    assert lib.attn_selftest_wait_timeout(20_000_000, None) == 1


def _gqa(lib, q=A, kp=A, vp=A, bt=A, sl=A, o=A, lse=A, B=2, Hq=8, Hkv=2, D=128, page=64, npages=4, maxp=2,
         scale=0.1, ws=A, ws_bytes=1 << 20):
    return lib.attn_decode_paged_gqa(q, kp, vp, bt, sl, o, lse, B, Hq, Hkv, D, page, npages, maxp, scale, ws,
                                     ws_bytes, None)


def test_gqa_decode_rejects_bad_arguments(lib):
    assert _gqa(lib, q=None) == 1
    assert _gqa(lib, vp=None) == 1
    assert _gqa(lib, kp=A + 8) == 1          # misaligned
    assert _gqa(lib, sl=A + 2) == 1
    assert _gqa(lib, Hq=6, Hkv=4) == 1       # Hq % Hkv
    assert _gqa(lib, B=0) == 1
    assert _gqa(lib, npages=0) == 1
    assert _gqa(lib, scale=0.0) == 1
    assert _gqa(lib, scale=float("nan")) == 1


def test_gqa_decode_unsupported_shapes(lib):
    assert _gqa(lib, D=96) == 2
    assert _gqa(lib, D=256) == 2
    assert _gqa(lib, Hq=32, Hkv=2) == 2      # group of 16
    assert _gqa(lib, page=16) == 2
    assert _gqa(lib, B=5000) == 2


def test_mtp_decode_argument_checks(lib):
    def call(B=2, s_q=2, Hq=128, Dk=576, Dv=512, page=64, q=A, scale=0.07):
        return lib.attn_decode_paged_mtp(q, A, A, A, A, A, B, s_q, Hq, Dk, Dv, page, 8, 4, scale, A, 1 << 20, None)
    assert call(q=None) == 1
    assert call(s_q=0) == 1
    assert call(scale=-1.0) == 1
    assert call(Hq=64) == 2
    assert call(B=1024, s_q=4) == 2          # more than 2048 query units
    assert lib.attn_decode_paged_mtp_workspace_size(1024, 4, 128, 512, 0) == 0


def test_bwd_argument_checks(lib):
    def call(q=A, lse=A, dk=A, B=1, Hq=4, Hkv=2, Nq=100, Nk=100, D=128, Dv=128, scale=0.1, ws=A, wsb=1 << 30):
        return lib.attn_bwd(q, A, A, A, A, lse, A, dk, A, B, Hq, Hkv, Nq, Nk, D, Dv, 1, scale, ws, wsb, None)
    assert call(q=None) == 1
    assert call(dk=None) == 1
    assert call(lse=A + 2) == 1              # misaligned
    assert call(Hq=6, Hkv=4) == 1            # Hq % Hkv
    assert call(B=0) == 1
    assert call(Nq=-1) == 1
    assert call(scale=0.0) == 1
    assert call(scale=float("inf")) == 1
    assert call(D=256, Dv=256) == 2          # dK and dV do not fit TMEM next to the work tiles
    assert call(D=128, Dv=64) == 2
    assert call(D=96, Dv=96) == 2
    assert call(ws=None) == 5
    assert call(wsb=1024) == 5
    assert call(ws=A + 16) == 5              # workspace must be 256-byte aligned
    assert call(Nq=0, Nk=0, q=None, dk=None, ws=None, wsb=0) == 0
    need = lib.attn_bwd_workspace_size(1, 4, 100, 128)
    assert need >= 100 * 4 * 128 * 4 + 100 * 4 * 4
    # D = 128 keeps dQ transposed, each head dim's row of queries padded to a
    # multiple of 32 (128 bytes) for the TMA adds: 100 -> 128 queries
    assert need == 4 * 128 * 128 * 4 + 1792
    assert lib.attn_bwd_workspace_size(1, 4, 100, 64) == 100 * 4 * 64 * 4 + 1792
    assert lib.attn_bwd_workspace_size(1, 4, 100, 256) == 0


def test_fwd_fp8_argument_checks(lib):
    def call(q=A, D=128, descale=0.01, scale=0.1, Hq=4, Hkv=2):
        return lib.attn_fwd_fp8(q, A, A, descale, 0.02, 0.03, A, A, 1, Hq, Hkv, 100, 100, D, 1, scale, None)
    assert call(q=None) == 1
    assert call(q=A + 8) == 1                # misaligned
    assert call(descale=0.0) == 1
    assert call(descale=float("nan")) == 1
    assert call(scale=-1.0) == 1
    assert call(Hq=6, Hkv=4) == 1
    assert call(D=64) == 2
    assert call(D=256) == 2


def test_workspace_sizes_reject_bad_device_index(lib):
    # the split plan depends on the SM count of the device the call will run on;
    # a device index that names no CUDA device gives 0 (no GPU is needed for this)
    for dev in (-1, 4096):
        assert lib.attn_decode_paged_workspace_size(64, 128, 512, dev) == 0
        assert lib.attn_decode_paged_mtp_workspace_size(64, 2, 128, 512, dev) == 0
        assert lib.attn_decode_paged_gqa_workspace_size(64, 32, 8, 128, dev) == 0
    # unsupported shapes give 0 whatever the device
    assert lib.attn_decode_paged_workspace_size(64, 64, 512, 0) == 0
    assert lib.attn_decode_paged_gqa_workspace_size(64, 32, 8, 96, 0) == 0
