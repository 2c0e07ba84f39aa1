"""CPU checks of the boundary: the library builds, loads and exports every
function include/albert.h declares; the Python binding's structs and status
codes agree with the header.  No compute call is made (no GPU here)."""
import ctypes as C
import os
import re

import pytest

import synth

import transformer_encoder_albert_b200 as tea
from transformer_encoder_albert_b200 import build as tea_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "albert.h")


def _header():
    with open(HEADER) as f:
        return f.read()


def _declared_functions():
    text = re.sub(r"/\*.*?\*/", "", _header(), flags=re.S)
    return sorted(set(re.findall(r"\b(albert_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    tea_build.build()
    return C.CDLL(tea.LIB_PATH)


def test_library_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert "albert_create" in names and "albert_forward" in names and "albert_destroy" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(tea.EXPORTS)


def test_status_codes_match_header():
    codes = dict((m[0], int(m[1])) for m in re.findall(r"#define (ALBERT_(?:OK|ERR_\w+))\s+(\d+)", _header()))
    for code, name in tea.STATUS_NAMES.items():
        assert codes[name] == code


def test_config_struct_matches_header_field_order():
    text = _header()
    body = re.search(r"typedef struct \{(.*?)\} albert_config;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"\b(\w+)\s*;", body)
    assert fields == [f for f, _ in tea.albert_config._fields_]
    assert C.sizeof(tea.albert_config) == 4 * len(fields)  # 4-byte ints and one float


def test_weights_struct_matches_header_field_order():
    body = re.search(r"typedef struct \{(.*?)\} albert_weights;", _header(), re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"\*\s*(\w+)", body)
    assert tuple(fields) == tea.WEIGHT_FIELDS


def test_library_is_built_for_sm100a_only():
    assert "arch=compute_100a,code=sm_100a" in " ".join(tea_build.FLAGS)


def test_host_side_rejections_need_no_gpu(lib):
    """Null pointers are rejected before any CUDA call."""
    lib.albert_create.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
    assert lib.albert_create(None, None, None) == 1
    h = C.c_void_p()
    assert lib.albert_create(None, None, C.byref(h)) == 1 and h.value is None
    lib.albert_forward.argtypes = [C.c_void_p] * 3 + [C.c_int, C.c_int, C.c_void_p, C.c_void_p]
    assert lib.albert_forward(None, None, None, 1, 1, None, None) == 1
    lib.albert_destroy.argtypes = [C.c_void_p]
    lib.albert_destroy(None)


def test_create_rejects_bad_group_counts_and_layouts_before_touching_the_device():
    """albert_create validates the config on the host first: these return
    ALBERT_ERR_CONFIG without any CUDA call (the weight pointers are never read)."""
    import transformer_encoder_albert_b200 as tea
    lib = tea.lib()
    dummy = tea.albert_weights(*([C.c_void_p(16)] * len(tea.WEIGHT_FIELDS)))
    for n_exec, n_groups, layout in ((12, 0, 0), (3, 4, 0), (0, 2, 0), (12, -1, 0), (12, 1, 2), (12, 1, -1)):
        cfg = tea.make_config(synth.ARCH, n_exec=n_exec, n_groups=n_groups, out_layout=layout)
        h = C.c_void_p()
        assert lib.albert_create(C.byref(dummy), C.byref(cfg), C.byref(h)) == 2  # ALBERT_ERR_CONFIG
        assert h.value is None


def _fake(addr=4096):
    """A non-NULL, 256-byte aligned pointer value that the host checks never dereference."""
    return C.c_void_p(addr)


def test_length_regulation_host_rejections_need_no_gpu(lib):
    """albert_length_regulate validates pointers, sizes, the speed and alignment on
    the host and returns before any CUDA call."""
    f = lib.albert_length_regulate
    f.argtypes = [C.c_void_p, C.c_int, C.c_float, C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]
    p = _fake()

    def call(logits=p, Cch=50, speed=1.0, feats=p, D=512, cu=p, nseq=2, n_tok=10, frames=p, max_frames=100,
             scratch=p):
        return f(logits, Cch, speed, feats, D, cu, nseq, n_tok, p, p, p, frames, max_frames, scratch, p, None)

    assert call(logits=None) == 1 and call(feats=None) == 1 and call(scratch=None) == 1
    for kw in ({"Cch": 0}, {"D": 0}, {"D": 12}, {"nseq": 0}, {"n_tok": 0}, {"max_frames": -1}):
        assert call(**kw) == 3, kw
    for speed in (0.0, -1.0, float("inf"), float("nan")):
        assert call(speed=speed) == 2, speed
    assert call(feats=_fake(4096 + 8)) == 2 and call(frames=_fake(4096 + 4)) == 2 and call(scratch=_fake(4100)) == 2
    sb = lib.albert_length_regulate_scratch_bytes
    sb.restype = C.c_size_t
    assert sb(0) == 0
    # local starts (int32, padded to 8 bytes) + block sums and block starts (int64 per 32 tokens)
    for n in (1, 31, 32, 33, 18797):
        assert sb(n) == ((n * 4 + 7) // 8) * 8 + 2 * 8 * ((n + 31) // 32), n


def test_single_kernel_entries_reject_bad_arguments_on_the_host(lib):
    p = _fake()
    g = lib.albert_test_gemm
    g.argtypes = [C.c_void_p] * 6 + [C.c_float, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int,
                                     C.c_void_p]
    assert g(None, p, p, p, p, p, 1e-12, p, p, 128, 256, 64, 0, None) == 1
    assert g(p, p, p, p, p, p, 1e-12, p, p, 0, 256, 64, 0, None) == 3         # M < 1
    assert g(p, p, p, p, p, p, 1e-12, p, p, 128, 200, 64, 0, None) == 3       # N not a tile multiple
    assert g(p, p, p, p, p, p, 1e-12, p, p, 128, 256, 100, 0, None) == 3      # K not a multiple of 64
    assert g(p, p, p, p, p, p, 1e-12, p, p, 128, 256, 64, 9, None) == 2       # no such epilogue
    assert g(p, p, p, p, p, p, 1e-12, p, p, 128, 256, 64, 16 | 32, None) == 2  # both variants forced
    assert g(p, p, p, None, p, p, 1e-12, p, p, 128, 768, 64, 2, None) == 2    # LN epilogue without R
    assert g(p, p, _fake(4100), p, p, p, 1e-12, p, p, 128, 256, 64, 0, None) == 2  # misaligned bias
    a = lib.albert_test_attention
    a.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p]
    assert a(None, p, 1, 16, p, 0, None) == 1
    assert a(p, p, 0, 16, p, 0, None) == 3 and a(p, p, 1, 513, p, 0, None) == 3
    assert a(p, p, 1, 16, p, 3, None) == 2
    n = lib.albert_gemm_residual_ln_noalloc
    n.argtypes = [C.c_void_p] * 6 + [C.c_float, C.c_void_p, C.c_int, C.c_int, C.c_void_p]
    assert n(None, p, p, p, p, p, 1e-12, p, 16, 768, None) == 1
    assert n(p, p, p, p, p, p, 1e-12, p, 2049, 768, None) == 3 and n(p, p, p, p, p, p, 1e-12, p, 16, 100, None) == 3
    assert n(p, p, _fake(4104), p, p, p, 1e-12, p, 16, 768, None) == 2
