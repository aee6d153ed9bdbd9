"""The C-ABI library loads, exports every symbol include/attn_b200.h declares, and
rejects bad arguments on the host before any CUDA call (so this runs without a GPU)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_b200.h")
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def declared_symbols():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b((?:attn|w4a16)_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from exact_attention_forward_11_b200 import build
    build.build()
    import exact_attention_forward_11_b200 as m
    return m


def test_header_declares_the_boundary():
    syms = declared_symbols()
    assert {"attn_fwd", "attn_fwd_fp8", "attn_quantize_fp8", "attn_get_device_status",
            "attn_status_string", "attn_abi_version"} <= set(syms)


def test_library_exports_every_declared_symbol(lib):
    so = lib.LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for s in declared_symbols():
        assert s in exported, s
    handle = ctypes.CDLL(so)
    for s in declared_symbols():
        assert getattr(handle, s) is not None
    # the binding wraps every declared symbol under the same name
    for s in declared_symbols():
        assert s in lib.SIGNATURES and callable(getattr(lib, s))


def test_status_strings_and_version(lib):
    assert lib.attn_abi_version() == 1
    assert lib.attn_status_string(0) == "ATTN_OK"
    assert lib.attn_status_string(5) == "ATTN_ERR_TIMEOUT"
    assert lib.attn_status_string(99) == "ATTN_UNKNOWN_STATUS"


FAKE = 0x100000  # 16-byte aligned, never dereferenced: validation fails first


def test_fwd_argument_validation(lib):
    f = lib.attn_fwd
    ok = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, H=1, N=8, d=64, scale=0.0, causal=0, dtype=0,
              stream=None)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"], a["scale"],
                 a["causal"], a["dtype"], a["stream"])
    assert call(q=None) == lib.ATTN_ERR_INVALID_ARG
    assert call(o=None) == lib.ATTN_ERR_INVALID_ARG
    assert call(N=0) == lib.ATTN_ERR_INVALID_ARG
    assert call(B=-1) == lib.ATTN_ERR_INVALID_ARG
    assert call(causal=2) == lib.ATTN_ERR_INVALID_ARG
    assert call(scale=float("nan")) == lib.ATTN_ERR_INVALID_ARG
    assert call(scale=float("inf")) == lib.ATTN_ERR_INVALID_ARG
    assert call(scale=-0.125) == lib.ATTN_ERR_INVALID_ARG    # only 0 selects the default
    assert call(B=1 << 16, H=1 << 10, N=1 << 10) == lib.ATTN_ERR_INVALID_ARG  # rows overflow int32
    assert call(d=96) == lib.ATTN_ERR_UNSUPPORTED
    assert call(d=256) == lib.ATTN_ERR_UNSUPPORTED
    assert call(dtype=1) == lib.ATTN_ERR_UNSUPPORTED
    assert call(k=FAKE + 2) == lib.ATTN_ERR_MISALIGNED
    assert call(lse=FAKE + 4) == lib.ATTN_ERR_MISALIGNED


def test_fp8_argument_validation(lib):
    f = lib.attn_fwd_fp8
    base = [FAKE] * 7 + [None, 1, 1, 8, 128, 0.0, 0, None]
    assert f(*base[:3], None, *base[4:]) == lib.ATTN_ERR_INVALID_ARG
    args = list(base)
    args[11] = 64
    assert f(*args) == lib.ATTN_ERR_UNSUPPORTED
    args = list(base)
    args[12] = -1.0
    assert f(*args) == lib.ATTN_ERR_INVALID_ARG
    args = list(base)
    args[2] = FAKE + 1
    assert f(*args) == lib.ATTN_ERR_MISALIGNED
    q = lib.attn_quantize_fp8
    assert q(None, None, FAKE, FAKE, 1, 1, 8, 128, None) == lib.ATTN_ERR_INVALID_ARG
    assert q(FAKE, None, FAKE, FAKE, 1, 1, 8, 64, None) == lib.ATTN_ERR_UNSUPPORTED
    assert q(FAKE, FAKE + 8, FAKE, FAKE, 1, 1, 8, 128, None) == lib.ATTN_ERR_MISALIGNED


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import exact_attention_forward_11_b200 as m
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(m, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        m.load()


def test_bwd_argument_validation(lib):
    f = lib.attn_bwd
    need = lib.attn_bwd_workspace_bytes(1, 2, 100, 128)
    assert need == 1024                       # 2 x 100 rows x 4 bytes, rounded up to 256
    assert lib.attn_bwd_workspace_bytes(1, 1, 8, 96) == 0
    assert lib.attn_bwd_workspace_bytes(0, 1, 8, 128) == 0
    ok = [FAKE] * 10 + [need, 1, 2, 100, 128, 0.0, 0, None]

    def call(i=None, val=None):
        a = list(ok)
        if i is not None:
            a[i] = val
        return f(*a)
    assert call(9, None) == lib.ATTN_ERR_INVALID_ARG           # no workspace
    assert call(10, need - 4) == lib.ATTN_ERR_INVALID_ARG      # workspace too small
    assert call(4, None) == lib.ATTN_ERR_INVALID_ARG           # no lse
    assert call(16, 3) == lib.ATTN_ERR_INVALID_ARG             # causal flag
    assert call(15, -1.0) == lib.ATTN_ERR_INVALID_ARG          # negative scale
    assert call(14, 96) == lib.ATTN_ERR_UNSUPPORTED
    assert call(6, FAKE + 8) == lib.ATTN_ERR_MISALIGNED
    assert call(9, FAKE + 4) == lib.ATTN_ERR_MISALIGNED


def test_w4a16_argument_validation(lib):
    f = lib.w4a16_gemm
    ok = [FAKE] * 5 + [16, 256, 512, None]

    def call(i=None, val=None):
        a = list(ok)
        if i is not None:
            a[i] = val
        return f(*a)
    assert call(1, None) == lib.ATTN_ERR_INVALID_ARG
    assert call(5, 0) == lib.ATTN_ERR_INVALID_ARG
    assert call(5, 129) == lib.ATTN_ERR_UNSUPPORTED       # M above 128
    assert call(6, 200) == lib.ATTN_ERR_UNSUPPORTED       # N not a multiple of 128
    assert call(7, 100) == lib.ATTN_ERR_UNSUPPORTED       # K not a multiple of 128
    assert call(4, FAKE + 2) == lib.ATTN_ERR_MISALIGNED


def test_w4a16_splitk_workspace_and_validation(lib):
    """Workspace size of the split-K W4A16 call: the tickets (16 bytes per 128
    columns, rounded up to 256) plus two fp32 slots of mpad x 128 values for each
    of at most 296 CTAs, one CTA per 8 slices for small problems; argument
    errors come back before any CUDA call."""
    wsb = lib.w4a16_gemm_splitk_workspace_bytes
    # decode MLP shape: 224 tiles x 64 slices -> 296 CTAs
    assert wsb(16, 28672, 8192) == 3584 + 2 * 296 * 16 * 128 * 4
    assert wsb(1, 28672, 8192) == wsb(16, 28672, 8192)            # M padded to 16
    assert wsb(17, 28672, 8192) == 3584 + 2 * 296 * 32 * 128 * 4
    # 8 tiles x 32 slices = 256 units -> 32 CTAs
    assert wsb(16, 1024, 4096) == 256 + 2 * 32 * 16 * 128 * 4
    # one unit -> one CTA
    assert wsb(128, 128, 128) == 256 + 2 * 1 * 128 * 128 * 4
    for bad in ((0, 128, 128), (129, 128, 128), (16, 200, 128), (16, 128, 100), (16, -128, 128)):
        assert wsb(*bad) == 0
    f = lib.w4a16_gemm_splitk
    need = wsb(16, 256, 512)
    ok = [FAKE] * 6 + [need, 16, 256, 512, None]

    def call(i=None, val=None):
        a = list(ok)
        if i is not None:
            a[i] = val
        return f(*a)
    assert call(5, None) == lib.ATTN_ERR_INVALID_ARG           # no workspace
    assert call(6, need - 16) == lib.ATTN_ERR_INVALID_ARG      # workspace too small
    assert call(5, FAKE + 8) == lib.ATTN_ERR_MISALIGNED
    assert call(1, None) == lib.ATTN_ERR_INVALID_ARG
    assert call(7, 129) == lib.ATTN_ERR_UNSUPPORTED
    assert call(8, 200) == lib.ATTN_ERR_UNSUPPORTED
    assert call(4, FAKE + 2) == lib.ATTN_ERR_MISALIGNED


def test_debug_build_exports_the_same_boundary(lib):
    """The debug build (-DATTN_DEBUG) builds, exports every declared symbol, says
    it is the debug build, and validates arguments on the host like the release
    build; the release build refuses the debug-only hook without touching CUDA."""
    from exact_attention_forward_11_b200 import build
    so = build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared_symbols()) <= exported
    assert lib.attn_debug_build() == 0
    assert lib.attn_status_string(6) == "ATTN_ERR_BOUNDS"
    assert lib.attn_fwd_debug_row_limit(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 64, 0.0, 0, 4, None) == \
        lib.ATTN_ERR_UNSUPPORTED
    prev = lib.use_library(lib.DEBUG_LIB_PATH)
    try:
        assert lib.attn_debug_build() == 1
        f = lib.attn_fwd_debug_row_limit
        assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 64, 0.0, 0, -1, None) == lib.ATTN_ERR_INVALID_ARG
        assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 64, 0.0, 0, 9, None) == lib.ATTN_ERR_INVALID_ARG
        assert f(None, FAKE, FAKE, FAKE, None, 1, 1, 8, 64, 0.0, 0, 4, None) == lib.ATTN_ERR_INVALID_ARG
        assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 96, 0.0, 0, 4, None) == lib.ATTN_ERR_UNSUPPORTED
        assert lib.attn_fwd(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 64, -1.0, 0, 0, None) == lib.ATTN_ERR_INVALID_ARG
    finally:
        lib.use_library(prev)
    assert lib.attn_debug_build() == 0
