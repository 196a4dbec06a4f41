"""The C ABI without a GPU: libfp8moe.so loads, exports every entry point
that include/moe.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import fp8_expert_ffn_b200 as fx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(moe_\w+)\s*\(", text, flags=re.M))


def test_header_declares_the_entry_points():
    names = header_functions()
    assert names == set(fx.ENTRY_POINTS), names ^ set(fx.ENTRY_POINTS)
    for required in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = fx.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", fx.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)$", out, flags=re.M))
    for name in header_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_status_strings():
    for code in range(7):
        s = fx.status_string(code)
        assert isinstance(s, str) and s
    assert fx.status_string(0) == "ok"
    assert fx.status_string(99) == "unknown status"


def _desc(**kw):
    d = dict(hidden=5120, n_routed=256, n_shared=1, top_k=8, ffn=1536, shared_ffn=1536, block=128,
             routed_scaling=1.0, norm_topk=1, n_group=1, topk_group=1)
    d.update(kw)
    return fx.moe_layer_desc(**d)


def _weights(ptr=4096, ld_h=5120, ld_f=1536, bias=None):
    return fx.moe_weights(ptr, ptr, ptr, ptr, ptr, ptr, ptr, ld_h, ld_f, bias)


def _create(desc, w):
    h = ctypes.c_void_p(1234)
    code = fx.lib().moe_layer_create(ctypes.byref(desc) if desc is not None else None,
                                     ctypes.byref(w) if w is not None else None, ctypes.byref(h))
    return code, h.value


@pytest.mark.parametrize("kw,code", [
    (dict(hidden=5000), fx.MOE_ERR_UNSUPPORTED),          # not a multiple of 128
    (dict(n_shared=2), fx.MOE_ERR_UNSUPPORTED),
    (dict(top_k=9), fx.MOE_ERR_UNSUPPORTED),
    (dict(n_routed=300), fx.MOE_ERR_UNSUPPORTED),
    (dict(shared_ffn=1024), fx.MOE_ERR_UNSUPPORTED),
    (dict(block=64), fx.MOE_ERR_UNSUPPORTED),
    (dict(norm_topk=2), fx.MOE_ERR_UNSUPPORTED),
    (dict(n_group=0), fx.MOE_ERR_UNSUPPORTED),
    (dict(n_group=3), fx.MOE_ERR_UNSUPPORTED),            # 256 experts do not split in 3
    (dict(n_group=64), fx.MOE_ERR_UNSUPPORTED),           # more than 32 groups
    (dict(n_group=8, topk_group=9), fx.MOE_ERR_UNSUPPORTED),
    (dict(n_group=8, topk_group=0), fx.MOE_ERR_UNSUPPORTED),
    (dict(n_routed=16, top_k=8, n_group=8, topk_group=3), fx.MOE_ERR_UNSUPPORTED),  # 3 groups of 2 < 8
    (dict(top_k=0), fx.MOE_ERR_INVALID_ARG),
    (dict(ffn=0, shared_ffn=0), fx.MOE_ERR_INVALID_ARG),
])
def test_create_rejects_bad_shapes(kw, code):
    c, h = _create(_desc(**kw), _weights())
    assert c == code and h is None


def test_create_rejects_bad_weights():
    assert _create(None, _weights())[0] == fx.MOE_ERR_INVALID_ARG
    assert _create(_desc(), None)[0] == fx.MOE_ERR_INVALID_ARG
    assert _create(_desc(), _weights(ptr=0))[0] == fx.MOE_ERR_INVALID_ARG
    assert _create(_desc(), _weights(ptr=4097))[0] == fx.MOE_ERR_MISALIGNED
    assert _create(_desc(), _weights(bias=4100))[0] == fx.MOE_ERR_MISALIGNED
    assert _create(_desc(), _weights(ld_h=5128))[0] == fx.MOE_ERR_MISALIGNED
    assert _create(_desc(), _weights(ld_h=4096))[0] == fx.MOE_ERR_INVALID_ARG
    assert _create(_desc(), _weights(ld_f=1500))[0] == fx.MOE_ERR_INVALID_ARG
    assert _create(_desc(ffn=1500, shared_ffn=1500), _weights(ld_f=1500))[0] == fx.MOE_ERR_MISALIGNED


def test_null_layer_everywhere():
    L = fx.lib()
    assert L.moe_workspace_size(None, 64) == 0
    assert L.moe_kernels_per_forward(None, 64) == 0
    assert L.moe_layer_destroy(None) == fx.MOE_OK
    assert L.moe_route(None, 16, 1, 5120, 16, 16, None, 16, 1 << 20, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_permute(None, 16, 1, 5120, 16, 16, 16, 16, 16, 16, 16, 1 << 20, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn(None, 16, 16, 16, 1, 16, 16, 1 << 20, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_gate_up(None, 16, 16, 16, 1, 16, 16, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_down(None, 16, 16, 16, 1, 16, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_combine(None, 16, 16, 16, 1, 16, 5120, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_layer_forward(None, 16, 1, 5120, 16, 5120, 16, 1 << 20, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_get_device_status(None, None, None) == fx.MOE_ERR_INVALID_ARG
    assert L.moe_test_grouped_gemm_f32(None, 0, 16, 16, 16, 1, 16, None) == fx.MOE_ERR_INVALID_ARG


CITES = ("Dots3NoteTextConfig", "PR #47844", "Dots3-Note", "dots-studio/dots3-note-prev", "Dots 3 Note Preview")
NO_COUNTERPART = ("no counterpart on the pages", "The pages describe no such call")


def test_every_declared_call_cites_its_passage():
    """The comment in front of each declaration cites the page passage that
    defines the operation, or says that the pages have no counterpart."""
    text = open(HEADER).read()
    for name in header_functions():
        at = re.search(r"^\s*(?:const\s+)?\w+\s*\*?\s*" + name + r"\s*\(", text, flags=re.M).start()
        end = text.rfind("*/", 0, at)
        comment = " ".join(text[text.rfind("/*", 0, end):end].replace("*", " ").split())
        assert any(c in comment for c in CITES + NO_COUNTERPART), f"{name}: no citation in {comment[:80]!r}"
