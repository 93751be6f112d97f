"""The C ABI without a GPU: the library loads, exports every declared entry point, its struct
layouts match the binding, and invalid arguments are rejected on the host before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

import head_scaled_dot_sdpa_b200 as sdpa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdpa.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"SDPA_API\s+[\w\s\*]+?\b(\w+)\(", text)


def test_every_declared_function_is_exported():
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(sdpa.lib, n), f"{n} declared in sdpa.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", sdpa.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(names) <= exported


def test_range_checked_build_differs_and_reports_itself():
    """libsdpa_debug.so is the same sources compiled with SDPA_DEBUG_CHECKS: it exports the same
    entry points, says so through sdpa_debug_checks(), and its kernels are different code."""
    debug = os.path.join(os.path.dirname(sdpa.LIB_PATH), "libsdpa_debug.so")
    normal = os.path.join(os.path.dirname(sdpa.LIB_PATH), "libsdpa.so")
    assert os.path.exists(debug), "build it with head_scaled_dot_sdpa_b200/build.py --debug-checks"
    libs = {path: ctypes.CDLL(path) for path in (normal, debug)}
    for lib in libs.values():
        lib.sdpa_debug_checks.restype = ctypes.c_int
        for n in declared_functions():
            assert hasattr(lib, n), n
    assert libs[normal].sdpa_debug_checks() == 0
    assert libs[debug].sdpa_debug_checks() == 1
    objs = os.path.join(ROOT, "_build")
    a = os.path.join(objs, "sdpa", "prefill_bf16_d128.cu.o")
    b = os.path.join(objs, "sdpa_debug", "prefill_bf16_d128.cu.o")
    if os.path.exists(a) and os.path.exists(b):
        assert open(a, "rb").read() != open(b, "rb").read()
    assert open(normal, "rb").read() != open(debug, "rb").read()


def test_struct_layout_matches_binding(tmp_path):
    src = tmp_path / "layout.c"
    fields = [f[0] for f in sdpa.Params._fields_]
    bfields = [f[0] for f in sdpa.BlockMaskInfoStruct._fields_]
    sfields = [f[0] for f in sdpa.PackedSegments._fields_]
    body = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', 'int main(void){']
    body.append('printf("%zu\\n", sizeof(sdpa_params));')
    body += [f'printf("%zu\\n", offsetof(sdpa_params, {f}));' for f in fields]
    body.append('printf("%zu\\n", sizeof(sdpa_block_mask_info));')
    body += [f'printf("%zu\\n", offsetof(sdpa_block_mask_info, {f}));' for f in bfields]
    body.append('printf("%zu\\n", sizeof(sdpa_packed_segments));')
    body += [f'printf("%zu\\n", offsetof(sdpa_packed_segments, {f}));' for f in sfields]
    body.append('return 0;}')
    src.write_text("\n".join(body))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-o", str(exe), str(src)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(sdpa.Params)] + [getattr(sdpa.Params, f).offset for f in fields]
    want += [ctypes.sizeof(sdpa.BlockMaskInfoStruct)] + [getattr(sdpa.BlockMaskInfoStruct, f).offset for f in bfields]
    want += [ctypes.sizeof(sdpa.PackedSegments)] + [getattr(sdpa.PackedSegments, f).offset for f in sfields]
    assert got == want


def _params(**kw):
    p = sdpa.Params()
    p.dtype, p.batch, p.q_len, p.kv_len = sdpa.SDPA_BF16, 2, 16, 16
    p.nheads, p.nkvheads, p.dqk, p.dv = 4, 2, 64, 64
    p.scale = float("nan")
    for k, v in kw.items():
        setattr(p, k, v)
    return p


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _forward(p, ws=FAKE, ws_bytes=1 << 30):
    return sdpa.lib.sdpa_forward(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code,words", [
    (dict(nkvheads=3), sdpa.SDPA_ERR_INVALID_ARG, "divisible"),
    (dict(dtype=7), sdpa.SDPA_ERR_INVALID_ARG, "dtype"),
    (dict(causal=5), sdpa.SDPA_ERR_INVALID_ARG, "causal"),
    (dict(dqk=0), sdpa.SDPA_ERR_INVALID_ARG, "positive"),
    (dict(batch=-1), sdpa.SDPA_ERR_INVALID_ARG, "negative"),
])
def test_invalid_params_rejected(kw, code, words):
    p = _params(**kw)
    assert _forward(p) == code
    assert words in sdpa.lib.sdpa_last_error().decode()
    assert sdpa.lib.sdpa_workspace_size(ctypes.byref(p)) == 0


def test_null_params():
    assert sdpa.lib.sdpa_forward(None, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == sdpa.SDPA_ERR_INVALID_ARG


def test_workspace_checks():
    p = _params()
    need = sdpa.lib.sdpa_workspace_size(ctypes.byref(p))
    assert need >= 256 and need % 256 == 0
    assert _forward(p, ws=None) == sdpa.SDPA_ERR_WORKSPACE
    assert _forward(p, ws=FAKE + 16) == sdpa.SDPA_ERR_WORKSPACE
    assert _forward(p, ws_bytes=need - 1) == sdpa.SDPA_ERR_WORKSPACE


def test_decode_workspace_holds_the_partials():
    p = _params(batch=64, q_len=1, kv_len=8192, nheads=32, nkvheads=8, dqk=128, dv=128,
                causal=sdpa.SDPA_CAUSAL_BOTTOM_RIGHT)
    need = sdpa.lib.sdpa_workspace_size(ctypes.byref(p))
    # at least one fp32 partial row of 128 per (batch, kv head, split of the capacity)
    assert need > 64 * 8 * 128 * 4


def test_decode_argument_rules():
    p = _params(q_len=1, causal=sdpa.SDPA_CAUSAL_TOP_LEFT)
    rc = sdpa.lib.sdpa_decode_with_cache(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                         FAKE, 1 << 30, None)
    assert rc == sdpa.SDPA_ERR_INVALID_ARG and "BOTTOM_RIGHT" in sdpa.lib.sdpa_last_error().decode()
    p = _params(q_len=1, causal=sdpa.SDPA_CAUSAL_BOTTOM_RIGHT, kv_lengths=FAKE)
    rc = sdpa.lib.sdpa_decode_with_cache(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                         FAKE, 1 << 30, None)
    assert rc == sdpa.SDPA_ERR_INVALID_ARG


def test_cache_update_rules():
    f = sdpa.lib.cache_update_at_index
    assert f(FAKE, FAKE, FAKE, FAKE, 9, 128, 8, 1, 16, 2, FAKE, None, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, sdpa.SDPA_BF16, 128, 8, 17, 16, 2, FAKE, None, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, sdpa.SDPA_BF16, 128, 8, 1, 16, 2, None, None, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(FAKE, None, FAKE, FAKE, sdpa.SDPA_BF16, 128, 8, 1, 16, 2, FAKE, None, None) == sdpa.SDPA_ERR_INVALID_ARG


def test_block_mask_info_sizes_and_rules():
    size = sdpa.lib.build_block_mask_info_size
    assert size(16, 16384, 16384, 128, 128) >= 16 * 128 * 128 * 128 * 4 * 4
    assert size(1, 10, 10, 4, 30) == 0       # bk not a multiple of 32
    assert size(1, 10, 10, 1024, 128) == 0   # more words per block than the kernel keeps
    st = sdpa.BlockMaskInfoStruct()
    strides = (ctypes.c_int64 * 3)(2, 256, 65536)
    rc = sdpa.lib.build_block_mask_info(FAKE, strides, 1, 256, 128, 128, 128, FAKE, 1 << 30,
                                        ctypes.byref(st), None)
    assert rc == sdpa.SDPA_ERR_INVALID_ARG and "mask_stride[0]" in sdpa.lib.sdpa_last_error().decode()


def test_block_info_must_match_the_call():
    st = sdpa.BlockMaskInfoStruct(nheads=4, q_len=16, kv_len=32, bq=128, bk=128, nqb=1, nkb=1,
                                  block_class=FAKE, row_count=FAKE, row_list=FAKE, partial_bits=FAKE)
    p = _params(block_info=ctypes.pointer(st))
    assert _forward(p) == sdpa.SDPA_ERR_INVALID_ARG
    assert "block_info" in sdpa.lib.sdpa_last_error().decode()


def _packed_call(p, seg, ws=FAKE, ws_bytes=1 << 30):
    return sdpa.lib.sdpa_forward_packed(ctypes.byref(p), None if seg is None else ctypes.byref(seg),
                                        FAKE, FAKE, FAKE, FAKE, ws, ws_bytes, None)


@pytest.mark.parametrize("pkw,skw,words", [
    (dict(batch=2), dict(), "batch must be 1"),
    (dict(bias=FAKE, bias_dtype=sdpa.SDPA_BF16), dict(), "not supported"),
    (dict(mask=FAKE), dict(), "not supported"),
    (dict(), dict(nseg=-1), "negative"),
    (dict(), dict(maxlen=-3), "negative"),
    (dict(), dict(q_segments=None), "q_segments is NULL"),
    (dict(), dict(nseg=0), "no segments"),
])
def test_packed_argument_rules(pkw, skw, words):
    """Packed sequences: no batch axis, no bias or mask, a segment vector for any rows."""
    p = _params(**{**dict(batch=1, q_len=300, kv_len=300), **pkw})
    seg = sdpa.PackedSegments(3, 200, FAKE, None)
    for k, v in skw.items():
        setattr(seg, k, v)
    assert _packed_call(p, seg) == sdpa.SDPA_ERR_INVALID_ARG
    assert words in sdpa.lib.sdpa_last_error().decode()
    assert sdpa.lib.sdpa_packed_workspace_size(ctypes.byref(p), ctypes.byref(seg)) == 0


def test_packed_workspace_holds_the_segment_starts():
    p = _params(batch=1, q_len=300, kv_len=300)
    assert _packed_call(p, None) == sdpa.SDPA_ERR_INVALID_ARG
    for nseg in (1, 63, 64, 5000):
        seg = sdpa.PackedSegments(nseg, 300, FAKE, None)
        need = sdpa.lib.sdpa_packed_workspace_size(ctypes.byref(p), ctypes.byref(seg))
        assert need % 256 == 0 and need >= 256 + 2 * 4 * (nseg + 1)
        assert _packed_call(p, seg, ws_bytes=need - 1) == sdpa.SDPA_ERR_WORKSPACE


def test_backward_argument_rules():
    """The fused gradient takes no bias and head sizes up to 256; its workspace holds two floats
    per query row and head."""
    p = _params(bias=FAKE, bias_dtype=sdpa.SDPA_BF16)
    rc = sdpa.lib.sdpa_backward(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                1 << 30, None)
    assert rc == sdpa.SDPA_ERR_INVALID_ARG and "bias" in sdpa.lib.sdpa_last_error().decode()
    p = _params(dqk=320, dv=64)
    rc = sdpa.lib.sdpa_backward(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                1 << 30, None)
    assert rc == sdpa.SDPA_ERR_UNSUPPORTED
    p = _params(batch=4, q_len=2048, nheads=32, nkvheads=8)
    need = sdpa.lib.sdpa_backward_workspace_size(ctypes.byref(p))
    assert need % 256 == 0 and need >= 256 + 4 * 2048 * 32 * 8
    rc = sdpa.lib.sdpa_backward(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                need - 1, None)
    assert rc == sdpa.SDPA_ERR_WORKSPACE


def test_with_weights_argument_rules():
    """A drop probability outside [0, 1) and v_head_dim above 256 are rejected on the host."""
    f = sdpa.lib.sdpa_forward_with_weights
    for bad in (-0.1, 1.0, float("nan")):
        p = _params()
        assert f(ctypes.byref(p), bad, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == sdpa.SDPA_ERR_INVALID_ARG
        assert "drop probability" in sdpa.lib.sdpa_last_error().decode()
    p = _params(dv=320)
    assert f(ctypes.byref(p), 0.0, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == sdpa.SDPA_ERR_UNSUPPORTED
    p = _params()
    assert f(ctypes.byref(p), 0.0, 0, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1 << 20, None) == sdpa.SDPA_ERR_WORKSPACE


def test_rope_argument_rules():
    """The rotary embedding needs an even head size, a positive base, and pointers when there
    are rows; zero rows is a no-op."""
    f = sdpa.lib.sdpa_rope
    assert f(FAKE, FAKE, sdpa.SDPA_BF16, 4, 2, 63, FAKE, 10000.0, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert "even head size" in sdpa.lib.sdpa_last_error().decode()
    assert f(FAKE, FAKE, sdpa.SDPA_BF16, 4, 2, 64, FAKE, 0.0, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 9, 4, 2, 64, FAKE, 10000.0, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(None, FAKE, sdpa.SDPA_BF16, 4, 2, 64, FAKE, 10000.0, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(None, None, sdpa.SDPA_BF16, 0, 2, 64, None, 10000.0, None) == sdpa.SDPA_OK
