"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects bad arguments before touching the GPU.  CPU only."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "attn_b200.h")


def _lib():
    from scaled_dot_product_prefill_b200 import _lib

    if not os.path.exists(_lib.lib_path()):
        from scaled_dot_product_prefill_b200 import build

        build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("attn_prefill", "attn_prefill_f32", "attn_decode_paged",
                     "attn_decode_paged_workspace_size", "attn_status_string", "attn_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = _lib()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in attn_b200.h but not exported"


def test_binding_prototypes_cover_the_header():
    from scaled_dot_product_prefill_b200 import _lib as L

    assert set(declared_functions()) == set(L.PROTOTYPES)


def test_status_strings_and_version():
    lib = _lib()
    assert lib.attn_status_string(0) == b"ATTN_OK"
    assert lib.attn_status_string(6) == b"ATTN_ERR_WORKSPACE"
    assert lib.attn_status_string(99) == b"ATTN_ERR_UNKNOWN"
    assert lib.attn_version() >= 100


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: every case below fails validation
MISALIGNED = ctypes.c_void_p(0x10008)


def prefill(lib, fn="attn_prefill", q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=1, Hq=4, Hkv=2, Sq=64, Skv=64, D=64,
            scale=0.125, causal=1, window=0):
    return getattr(lib, fn)(q, k, v, o, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, None)


@pytest.mark.parametrize("fn", ["attn_prefill", "attn_prefill_f32"])
def test_prefill_argument_validation(fn):
    lib = _lib()
    assert prefill(lib, fn, q=None) == 1
    assert prefill(lib, fn, o=MISALIGNED) == 1
    assert prefill(lib, fn, Hq=6, Hkv=4) == 1           # Hq not a multiple of Hkv
    assert prefill(lib, fn, Hkv=0) == 1
    assert prefill(lib, fn, Sq=-1) == 1
    assert prefill(lib, fn, scale=0.0) == 1
    assert prefill(lib, fn, scale=float("nan")) == 1
    assert prefill(lib, fn, causal=2) == 1
    assert prefill(lib, fn, window=-3) == 1
    assert prefill(lib, fn, D=96) == 1                  # head dim outside {64, 128}
    assert prefill(lib, fn, causal=0, window=16) == 2   # a window is a causal look-back
    # empty problems are no-ops, even with null pointers
    assert prefill(lib, fn, q=None, k=None, v=None, o=None, B=0) == 0
    assert prefill(lib, fn, q=None, k=None, v=None, o=None, Sq=0) == 0


def decode(lib, q=FAKE, kp=FAKE, vp=FAKE, pt=FAKE, sl=FAKE, page=16, N=4, Hq=8, Hkv=2, D=128, num_pages=64,
           max_pages=16, max_seq_len=256, scale=0.1, window=0, ws=FAKE, ws_bytes=1 << 30, out=FAKE):
    return lib.attn_decode_paged(q, kp, vp, pt, sl, page, N, Hq, Hkv, D, num_pages, max_pages, max_seq_len,
                                 scale, window, ws, ws_bytes, out, None)


def test_decode_argument_validation():
    lib = _lib()
    assert decode(lib, q=None) == 1
    assert decode(lib, kp=None) == 1
    assert decode(lib, Hq=8, Hkv=3) == 1
    assert decode(lib, kp=MISALIGNED) == 1
    assert decode(lib, scale=-1.0) == 1
    assert decode(lib, D=96) == 1
    assert decode(lib, Hq=24, Hkv=2) == 2               # group of 12
    assert decode(lib, Hq=32, Hkv=2) == 2               # group of 16
    assert decode(lib, page=8) == 2
    assert decode(lib, ws=None) == 6
    need = lib.attn_decode_paged_workspace_size(4, 8, 128, 256, 16)
    assert need > 0
    assert decode(lib, ws_bytes=need - 1) == 6
    assert decode(lib, N=0, q=None, out=None) == 0


def test_workspace_size_is_monotone_and_rejects_bad_sizes():
    lib = _lib()
    a = lib.attn_decode_paged_workspace_size(64, 32, 128, 8192, 16)
    b = lib.attn_decode_paged_workspace_size(64, 32, 128, 16384, 16)
    assert 0 < a < b
    assert lib.attn_decode_paged_workspace_size(-1, 32, 128, 8192, 16) == 0
    # partial outputs and log-sum-exps: N * Hq * splits * (D + 1) floats, between one split per
    # 1024 keys (the longest split) and one per 64 keys (the shortest)
    assert 64 * 32 * (8192 // 1024) * 129 * 4 <= a <= 64 * 32 * (8192 // 64) * 129 * 4 + 256


def test_oracle_is_not_imported_by_the_library():
    import sys

    for mod in [m for m in list(sys.modules) if m.startswith("scaled_dot_product_prefill_b200")]:
        src = getattr(sys.modules[mod], "__file__", None)
        if src and src.endswith(".py"):
            text = open(src).read()
            assert "import oracle" not in text and "from oracle" not in text, src


@pytest.mark.parametrize("fn", ["attn_prefill_lse", "attn_prefill_f32_lse"])
def test_prefill_lse_argument_validation(fn):
    lib = _lib()
    call = lambda lse, **kw: getattr(lib, fn)(FAKE, FAKE, FAKE, FAKE, lse, kw.get("B", 1), 4, 2, 64, 64,
                                              kw.get("D", 64), 0.125, 1, 0, None)
    assert call(None) == 1                        # the lse output is required
    assert call(ctypes.c_void_p(0x10002)) == 1    # misaligned lse
    assert call(FAKE, D=96) == 1
    assert call(None, B=0) == 0                   # empty problem


def test_paged_prefill_argument_validation():
    lib = _lib()

    def call(page=16, D=128, lse=None, window=0, causal=1, Hq=8, Hkv=2, q=FAKE, msl=256):
        return lib.attn_prefill_paged(q, FAKE, FAKE, FAKE, FAKE, page, 2, Hq, Hkv, 64, D, 64, 16, msl, 0.1, causal,
                                      window, FAKE, lse, None)
    assert call(q=None) == 1
    assert call(Hq=8, Hkv=3) == 1
    assert call(lse=ctypes.c_void_p(0x10002)) == 1
    assert call(page=8) == 2
    assert call(page=48) == 2
    assert call(D=96) == 1
    assert call(causal=0, window=16) == 2


def test_kv_append_argument_validation():
    lib = _lib()

    def call(kn=FAKE, kp=FAKE, pt=FAKE, sl=FAKE, page=16, B=2, Hkv=2, S=4, D=128, num_pages=8, max_pages=4):
        return lib.attn_kv_append(kn, FAKE, kp, FAKE, pt, sl, page, B, Hkv, S, D, num_pages, max_pages, None)
    assert call(kn=None) == 1
    assert call(kp=MISALIGNED) == 1
    assert call(sl=ctypes.c_void_p(0x10002)) == 1
    assert call(num_pages=0) == 1
    assert call(S=-1) == 1
    assert call(D=100) == 2              # rows must be whole 16-byte pieces
    assert call(page=12) == 2
    assert call(D=1024) == 2
    assert call(kn=None, kp=None, pt=None, sl=None, B=0) == 0      # nothing to append
    assert call(kn=None, kp=None, pt=None, sl=None, S=0) == 0
    assert lib.attn_status_string(7) == b"ATTN_ERR_OUT_OF_PAGES"


def test_library_needs_no_cxx_runtime_and_loads_first():
    """The .so depends on the C library alone, and loads in a process that has loaded nothing else.

    A C++ runtime pulled in by a late dlopen can fail for want of static TLS;
    the library avoids needing one at all.
    """
    import subprocess
    import sys

    from scaled_dot_product_prefill_b200 import _lib as L

    _lib()
    path = L.lib_path()
    with open(path, "rb") as f:
        data = f.read()
    for name in (b"libstdc++.so", b"libgcc_s.so"):
        assert name not in data, f"{path} references {name.decode()}"
    code = f"import ctypes; lib = ctypes.CDLL({path!r}); print(lib.attn_version())"
    out = subprocess.run([sys.executable, "-S", "-c", code], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert int(out.stdout.strip()) >= 100


def test_fp8_decode_argument_validation():
    lib = _lib()

    def call(ks=0.5, vs=0.5, D=128, Hq=8, Hkv=2, ws=FAKE, kp=FAKE):
        return lib.attn_decode_paged_fp8(FAKE, kp, FAKE, FAKE, FAKE, 16, 4, Hq, Hkv, D, 64, 16, 256, 0.1, ks, vs, 0,
                                         ws, 1 << 30, FAKE, None)
    assert call(ks=0.0) == 1
    assert call(vs=-1.0) == 1
    assert call(ks=float("nan")) == 1
    assert call(kp=None) == 1
    assert call(kp=MISALIGNED) == 1
    assert call(D=96) == 1
    assert call(Hq=24, Hkv=2) == 2
    assert call(ws=None) == 6


def test_fp8_append_argument_validation():
    lib = _lib()

    def call(ks=0.5, vs=0.5, D=128, kp=FAKE):
        return lib.attn_kv_append_fp8(FAKE, FAKE, kp, FAKE, FAKE, FAKE, 16, 2, 2, 4, D, 8, 4, ks, vs, None)
    assert call(ks=0.0) == 1
    assert call(vs=float("inf")) == 1
    assert call(kp=None) == 1
    assert call(D=100) == 2


def test_selftest_timeout_argument_validation():
    lib = _lib()
    assert lib.attn_selftest_wait_timeout(0, None) == 1
    assert lib.attn_selftest_wait_timeout(1001, None) == 1


@pytest.mark.parametrize("fn", ["attn_prefill", "attn_prefill_f32"])
def test_prefill_without_keys_accepts_null_k_and_v(fn):
    lib = _lib()
    # Skv == 0: k and v are never read; the call then needs the GPU to write zeros, so on a
    # machine without one it gets past validation and fails at the CUDA call, not as INVALID_ARG
    st = prefill(lib, fn, k=None, v=None, Skv=0)
    assert st in (0, 3)
    assert prefill(lib, fn, k=None, v=None, Skv=16) == 1


def test_host_prefill_argument_validation():
    lib = _lib()

    def call(qh=FAKE, kh=FAKE, vh=FAKE, oh=FAKE, qd=FAKE, kd=FAKE, vd=FAKE, od=FAKE, B=2, Hq=4, Hkv=2, D=64,
             chunks=0, Skv=64):
        return lib.attn_prefill_host(qh, kh, vh, oh, qd, kd, vd, od, B, Hq, Hkv, 64, Skv, D, 0.125, 1, 0, chunks,
                                     None, None, None)

    assert call(qh=None) == 1                    # host buffers are required
    assert call(oh=None) == 1
    assert call(od=None) == 1                    # and the device ones
    assert call(qd=MISALIGNED) == 1
    assert call(chunks=-1) == 1
    assert call(chunks=5) == 1                   # more pieces than (batch, kv head) pairs (2 x 2)
    assert call(D=96) == 1
    assert call(B=0, qh=None, oh=None, qd=None, od=None) == 0   # empty problem


def test_host_decode_step_argument_validation():
    lib = _lib()

    def call(qh=FAKE, kh=FAKE, oh=FAKE, qd=FAKE, kd=FAKE, N=4, Hq=8, Hkv=2, D=128, page=16, ws=FAKE, msl=256):
        return lib.attn_decode_step_host(qh, kh, FAKE, oh, qd, kd, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, page, N, Hq,
                                         Hkv, D, 64, 16, msl, 0.1, 0, ws, 1 << 30, None)
    assert call(qh=None) == 1                    # host buffers are required
    assert call(oh=None) == 1
    assert call(kd=None) == 1                    # and the device ones
    assert call(kd=MISALIGNED) == 1
    assert call(D=96) == 1
    assert call(Hq=24, Hkv=2) == 2               # group of 12
    assert call(ws=None) == 6
    assert call(msl=0) == 1                      # no room to append the new token
    assert call(N=0, qh=None, oh=None) == 0      # empty batch
