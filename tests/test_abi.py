"""The C-ABI library loads on a machine without a GPU, exports every
function include/sink_attn.h declares, and rejects bad arguments on the host
before touching the device.  CPU only: no call here launches a kernel."""
import ctypes
import os
import re

import pytest

from sink_sliding_window_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sink_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sink_attn_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "sink_attn_fwd" in names and "sink_attn_bwd" in names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/sink_attn.h but not exported"
    assert set(ops.EXPORTS) <= set(names)


def test_header_is_c_and_links(L, tmp_path):
    """include/sink_attn.h is plain C (C99, pedantic, warnings as errors),
    and a C program that takes the address of every declared function links
    against the built library."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    names = declared_functions()
    body = "\n".join(f"  (void)&{n};" for n in names)
    src = tmp_path / "abi_check.c"
    src.write_text(f'#include "sink_attn.h"\nint main(void) {{\n{body}\n  return 0;\n}}\n')
    lib_dir = os.path.dirname(ops.lib_path())
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(tmp_path / "abi_check"), "-L", lib_dir, "-l:" + os.path.basename(ops.lib_path()),
           f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_status_strings(L):
    for code in range(8):
        s = ops.status_string(code)
        assert isinstance(s, str) and s
    assert ops.status_string(99) == "unknown status"


def dims(**kw):
    base = dict(T=256, Hq=8, Hkv=2, D=64, batch=2, max_seqlen=128)
    base.update(kw)
    return ops.make_dims(base["T"], base["Hq"], base["Hkv"], base["D"], base["batch"], base["max_seqlen"])


FAKE = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced: validation fails first


FWD_ENTRIES = ("sink_attn_fwd", "sink_attn_fwd_pair")


def call_fwd(L, d, q=FAKE, k=FAKE, v=FAKE, sinks=FAKE, cu=None, window=0, scale=0.125, out=FAKE, lse=FAKE,
             entry="sink_attn_fwd"):
    return getattr(L, entry)(ctypes.byref(d), q, k, v, sinks, cu, window, scale, out, lse, None)


@pytest.mark.parametrize("bad,code", [
    (dict(D=128), 4),            # only D = 64
    (dict(Hq=6, Hkv=4), 2),      # Hq % Hkv != 0
    (dict(Hq=12, Hkv=4), 4),     # G = 3 is not a power of two
    (dict(T=255), 2),            # uniform batch: T != B * S
    (dict(T=-1), 2),
    (dict(Hkv=0), 2),
    (dict(batch=0, max_seqlen=0), 2),
])
@pytest.mark.parametrize("entry", FWD_ENTRIES)
def test_fwd_rejects_bad_shapes(L, bad, code, entry):
    assert call_fwd(L, dims(**bad), entry=entry) == code


@pytest.mark.parametrize("entry", FWD_ENTRIES)
def test_fwd_rejects_null_and_misaligned(L, entry):
    assert getattr(L, entry)(None, FAKE, FAKE, FAKE, FAKE, None, 0, 0.125, FAKE, FAKE, None) == 1
    assert call_fwd(L, dims(), q=None, entry=entry) == 1
    assert call_fwd(L, dims(), lse=None, entry=entry) == 1
    assert call_fwd(L, dims(), k=ctypes.c_void_p((1 << 20) + 8), entry=entry) == 3
    assert call_fwd(L, dims(), out=ctypes.c_void_p((1 << 20) + 2), entry=entry) == 3


@pytest.mark.parametrize("entry", FWD_ENTRIES)
def test_fwd_rejects_bad_scale(L, entry):
    for s in (0.0, -0.125, float("inf"), float("nan")):
        assert call_fwd(L, dims(), scale=s, entry=entry) == 4


@pytest.mark.parametrize("entry", FWD_ENTRIES)
def test_fwd_empty_is_noop(L, entry):
    # T = 0: valid, nothing to do, no pointer is touched.
    assert call_fwd(L, dims(T=0, batch=0, max_seqlen=0), q=None, k=None, v=None, out=None, lse=None,
                    entry=entry) == 0


def test_fwd_with_rejects_unknown_kernel(L):
    # kernel ids other than SINK_ATTN_FWD_AUTO .. SINK_ATTN_FWD_CTA_PAIR: SINK_ATTN_ERR_UNSUPPORTED
    for kid in (-1, 4, 99):
        assert L.sink_attn_fwd_with(ctypes.byref(dims()), FAKE, FAKE, FAKE, FAKE, None, 0, 0.125, FAKE, FAKE, kid,
                                    None) == 4
    # and the same validation as sink_attn_fwd for a known id
    assert L.sink_attn_fwd_with(ctypes.byref(dims(D=128)), FAKE, FAKE, FAKE, FAKE, None, 0, 0.125, FAKE, FAKE, 2,
                                None) == 4
    assert L.sink_attn_fwd_with(ctypes.byref(dims()), None, FAKE, FAKE, FAKE, None, 0, 0.125, FAKE, FAKE, 3,
                                None) == 1


def test_fwd_binding_rejects_unknown_kernel_name():
    with pytest.raises(ValueError):
        ops.fwd(None, None, None, None, kernel="bogus")


def test_fwd_kernel_for(L):
    for window in (0, 1, 128, 4096):
        assert L.sink_attn_fwd_kernel_for(ctypes.byref(dims()), window) in (1, 2, 3)
    assert L.sink_attn_fwd_kernel_for(ctypes.byref(dims(D=32)), 0) == -1
    assert ops.fwd_kernel_for(256, 8, 2, 64, 2, 128, 0) in ("one_tile", "two_tiles", "pair")


def test_bwd_workspace_and_validation(L):
    d = dims()
    ws = L.sink_attn_bwd_workspace_size(ctypes.byref(d))
    assert ws > 0
    assert L.sink_attn_bwd_workspace_size(ctypes.byref(dims(D=32))) == 0
    # q, k, v, sinks, cu_seqlens, window, scale, out, lse, dout, dq, dk, dv, dsinks
    args = [FAKE] * 4 + [None, 0, ctypes.c_float(0.125)] + [FAKE] * 7
    # workspace too small
    assert L.sink_attn_bwd(ctypes.byref(d), *args, FAKE, ctypes.c_size_t(ws - 1), None) == 7
    assert L.sink_attn_bwd(ctypes.byref(d), *args, None, ctypes.c_size_t(ws), None) == 7
    # workspace misaligned
    assert L.sink_attn_bwd(ctypes.byref(d), *args, ctypes.c_void_p((1 << 20) + 16), ctypes.c_size_t(ws), None) == 3
    # dsinks NULL
    a2 = list(args)
    a2[13] = None
    assert L.sink_attn_bwd(ctypes.byref(d), *a2, FAKE, ctypes.c_size_t(ws), None) == 1


def test_launch_counts(L):
    assert L.sink_attn_fwd_launches(ctypes.byref(dims())) == 1
    assert L.sink_attn_fwd_launches(ctypes.byref(dims(T=0, batch=0, max_seqlen=0))) == 0
    assert L.sink_attn_bwd_launches(ctypes.byref(dims())) >= 0


def ddims(B=4, Lq=1, C=256, max_seqlen=257, Hq=64, Hkv=8, D=64):
    return ops.decode_dims(B, Lq, C, max_seqlen, Hq, Hkv, D)


def call_decode(L, d, ptrs=None, window=0, scale=0.125, ws=FAKE, ws_bytes=1 << 30):
    # q, k_new, v_new, k_cache, v_cache, cache_seqlens, sinks, window, scale, out, lse, workspace, bytes, stream
    p = [FAKE] * 7 if ptrs is None else ptrs
    return L.sink_attn_decode(ctypes.byref(d), *p[:7], int(window), ctypes.c_float(scale), FAKE, FAKE, ws,
                              ctypes.c_size_t(ws_bytes), None)


def test_decode_workspace_size(L):
    w = ops.decode_workspace_size(4, 1, 8192, 8192, 64, 8)
    assert w > 0 and w % 256 == 0
    # Partials for at least one split of 64 query rows x 64 dims per (sequence, kv head).
    assert w >= 4 * 8 * 64 * 64 * 4
    assert ops.decode_workspace_size(4, 1, 8192, 8192, 64, 8, D=32) == 0
    assert ops.decode_workspace_size(4, 9, 8192, 8192, 64, 8) == 0  # G * Lq = 72 > 64


@pytest.mark.parametrize("bad,code", [
    (dict(Lq=0), 2), (dict(C=0), 2), (dict(B=-1), 2), (dict(max_seqlen=0), 2), (dict(Hq=63), 2),
    (dict(D=128), 4), (dict(Hq=48, Hkv=8), 4), (dict(Lq=9), 4),
])
def test_decode_rejects_bad_sizes(L, bad, code):
    assert call_decode(L, ddims(**bad)) == code


def test_decode_rejects_bad_pointers_scale_and_workspace(L):
    d = ddims()
    for i in range(7):
        p = [FAKE] * 7
        p[i] = None
        assert call_decode(L, d, p) == 1, i
    p = [FAKE] * 7
    p[3] = ctypes.c_void_p((1 << 20) + 8)  # k_cache misaligned
    assert call_decode(L, d, p) == 3
    assert call_decode(L, d, scale=0.0) == 4
    need = ops.decode_workspace_size(4, 1, 256, 257, 64, 8)
    assert call_decode(L, d, ws_bytes=need - 1) == 7
    assert call_decode(L, d, ws=None) == 7


def test_decode_empty_batch_is_noop(L):
    assert call_decode(L, ddims(B=0), [None] * 7, ws=None, ws_bytes=0) == 0
    assert ops.decode_launches(0, 1, 256, 257, 64, 8) == 0
    assert ops.decode_launches(4, 1, 256, 257, 64, 8) == 3
    # One CTA per (sequence, key/value head) covers the cache (64 x 8 CTAs
    # already fill the grid; the split plan keeps one): the attention kernel
    # finishes the rows and the combine launch is skipped.
    assert ops.decode_launches(64, 1, 256, 257, 64, 8) == 2
    assert ops.decode_launches(64, 1, 128, 8192, 64, 8, window=128) == 2
    # A long cache is split over several CTAs and combined.
    assert ops.decode_launches(64, 1, 8192, 8192, 64, 8) == 3


def test_binding_refuses_host_tensors():
    """The binding passes device pointers only: a host tensor is refused
    before any call into the library (its address would otherwise reach the
    kernels as device memory)."""
    import torch
    from sink_sliding_window_b200 import ops
    with pytest.raises(ValueError):
        ops._ptr(torch.zeros(4))
    assert ops._ptr(None) is None
