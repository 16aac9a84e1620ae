"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host (no kernel is launched by these tests)."""
import ctypes
import os
import re

import pytest

from transformer_decode_persistent_b200 import build as B
from transformer_decode_persistent_b200 import kie as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kie.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return K.lib()


def header_symbols():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(kie_[a-z_]+)\s*\(", txt)))


def test_header_declares_the_boundary():
    syms = header_symbols()
    for s in ["kie_create", "kie_load_weights", "kie_prefill", "kie_decode", "kie_reset",
              "kie_destroy", "kie_last_error", "kie_position"]:
        assert s in syms
    assert sorted(K.EXPORTS) == syms


def test_library_exports_every_declared_symbol(L):
    for s in header_symbols():
        assert hasattr(L, s), s
    out = os.popen(f"nm -D --defined-only {K.LIB_PATH}").read()
    for s in header_symbols():
        assert re.search(rf"\bT {s}\b", out), f"{s} not exported"


def test_struct_layouts_match_header():
    # sizes from the C declarations (LP64): config 12*4 + 2*4; tensor 8+8+16+4(+4 pad);
    # opts 8*3 + 4*3 (+4 pad) + 8 + 4 + 4 (temperature) + 4 (top_k) + 4 (top_p) (+4 pad)
    # + 8 (seed); info 6*4 + 4*8
    assert ctypes.sizeof(K.kie_config) == 56
    assert ctypes.sizeof(K.kie_tensor) == 40
    assert ctypes.sizeof(K.kie_decode_opts) == 72
    assert ctypes.sizeof(K.kie_info) == 56
    # plan: shape 4*4; range 8 + 2*4; info 2*4 + 8 + 9*16
    assert ctypes.sizeof(K.kie_seg_shape) == 16
    assert ctypes.sizeof(K.kie_seg_range) == 16
    assert ctypes.sizeof(K.kie_plan_info) == 160


def _cfg(**kw):
    base = dict(n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, ffn=1024,
                vocab=4096, n_experts=0, top_k=0, ffn_expert=0, ffn_shared=0, max_ctx=64,
                rms_eps=1e-5, rope_theta=10000.0)
    base.update(kw)
    return K.kie_config(**base)


@pytest.mark.parametrize("bad", [dict(d_model=100), dict(head_dim=96), dict(n_kv_heads=8),
                                 dict(n_heads=40, n_kv_heads=2), dict(max_ctx=0),
                                 dict(ffn=0), dict(n_experts=4, top_k=5, ffn=0, ffn_expert=64,
                                                   ffn_shared=64),
                                 dict(rope_theta=0.0)])
def test_create_rejects_bad_shapes_on_host(L, bad):
    h = ctypes.c_void_p()
    st = L.kie_create(ctypes.byref(_cfg(**bad)), 0, ctypes.byref(h))
    assert st == -1 and not h.value
    assert L.kie_last_error(None)


def test_null_arguments(L):
    assert L.kie_create(None, 0, None) == -1
    assert L.kie_destroy(None) == 0
    assert L.kie_position(None) == -1
    assert L.kie_pending(None) == -1
    assert L.kie_reset(None) == -1
    assert L.kie_decode(None, 1, None, None, None) == -1
    assert L.kie_prefill(None, None, 1, None) == -1
    assert L.kie_get_info(None, None) == -1
    assert L.kie_rewind(None, 0, 0) == -1


def test_create_without_gpu_fails_cleanly(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    st = L.kie_create(ctypes.byref(_cfg()), 0, ctypes.byref(h))
    assert st == -1 and b"device" in L.kie_last_error(None)


def test_struct_layouts_match_a_c_compiler(tmp_path):
    # compile the header with gcc and compare every field offset with ctypes
    src = tmp_path / "layout.c"
    fields = {"kie_config": K.kie_config, "kie_tensor": K.kie_tensor,
              "kie_decode_opts": K.kie_decode_opts, "kie_info": K.kie_info}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "kie.h"', "int main(void){"]
    for sname, cls in fields.items():
        lines.append(f'printf("{sname} %zu\\n", sizeof({sname}));')
        for f, _ in cls._fields_:
            lines.append(f'printf("{sname}.{f} %zu\\n", offsetof({sname}, {f}));')
    lines.append("return 0;}")
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    assert os.system(f"gcc -I{ROOT}/include -o {exe} {src}") == 0
    got = dict(l.split() for l in os.popen(str(exe)).read().splitlines())
    for sname, cls in fields.items():
        assert int(got[sname]) == ctypes.sizeof(cls)
        for f, _ in cls._fields_:
            assert int(got[f"{sname}.{f}"]) == getattr(cls, f).offset, (sname, f)
