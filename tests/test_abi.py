"""The C ABI without a GPU: the library builds and loads, exports every function the headers
declare, the Python struct layouts match the C ones, and host-side validation rejects bad
arguments before any CUDA call."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import vision_transformer_encoder_fwd_b200 as V

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("vit.h", "vit_stages.h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(vit_\w+)\s*\(", src):
            names.add(m.group(1))
    return names


def test_library_builds_and_exports_all_declared_symbols():
    lib = V.load_library()
    names = declared_functions()
    assert {"vit_create", "vit_forward", "vit_seg_zero_shot", "vit_destroy", "vit_stage_linear"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", V.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (vit_\w+)", out))
    assert names <= exported, names - exported
    for n in names:
        assert hasattr(lib, n)


def test_struct_layouts_match_c():
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "vit.h"
int main(void) {
  printf("%zu %zu %zu %zu\n", sizeof(vit_config), sizeof(vit_block_weights), sizeof(vit_weights), sizeof(vit_outputs));
  printf("%zu %zu %zu %zu\n", offsetof(vit_config, ln_eps), offsetof(vit_outputs, patch_fp32),
         offsetof(vit_outputs, taps), offsetof(vit_outputs, hidden));
  printf("%zu %zu %zu %zu\n", sizeof(vit_dense_head_weights), offsetof(vit_dense_head_weights, bn_w),
         offsetof(vit_dense_head_weights, cv2_w), offsetof(vit_dense_head_weights, pred_b));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "p.c")
        open(c, "w").write(prog)
        exe = os.path.join(d, "p")
        subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    sizes = [int(x) for x in lines[0].split()]
    offs = [int(x) for x in lines[1].split()]
    assert sizes == [ctypes.sizeof(V.VitConfig), ctypes.sizeof(V.VitBlockWeights), ctypes.sizeof(V.VitWeights),
                     ctypes.sizeof(V.VitOutputs)]
    assert offs == [V.VitConfig.ln_eps.offset, V.VitOutputs.patch_fp32.offset, V.VitOutputs.taps.offset,
                    V.VitOutputs.hidden.offset]
    dense = [int(x) for x in lines[2].split()]
    D = V.VitDenseHeadWeights
    assert dense == [ctypes.sizeof(D), D.bn_w.offset, D.cv2_w.offset, D.pred_b.offset]


def _cfg(**kw):
    base = dict(patch=16, img_h=336, img_w=336, dim=384, depth=12, heads=6, mlp_dim=1536, n_registers=4,
                pos_on_cls=0, max_batch=1, ln_eps=1e-6, tap_mask=0)
    base.update(kw)
    return V.VitConfig(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(dim=320, heads=5), V.VIT_E_UNSUPPORTED),          # not a multiple of 128
    (dict(heads=4), V.VIT_E_UNSUPPORTED),                   # head width != 64
    (dict(img_h=330), V.VIT_E_SHAPE),                        # not a multiple of the patch
    (dict(max_batch=0), V.VIT_E_INVALID_ARG),
    (dict(tap_mask=1 << 12), V.VIT_E_INVALID_ARG),           # tap after block 13 of 12
    (dict(tap_mask=0b11111), V.VIT_E_INVALID_ARG),           # five taps
    (dict(ln_eps=0.0), V.VIT_E_INVALID_ARG),
])
def test_create_rejects_bad_config_before_cuda(kw, expect):
    lib = V.load_library()
    h = ctypes.c_void_p()
    st = lib.vit_create(ctypes.byref(_cfg(**kw)), None, ctypes.byref(h))
    assert st == expect and not h.value
    assert lib.vit_last_error()


def test_create_rejects_missing_weights():
    lib = V.load_library()
    h = ctypes.c_void_p()
    assert lib.vit_create(ctypes.byref(_cfg()), ctypes.byref(V.VitWeights()), ctypes.byref(h)) == V.VIT_E_INVALID_ARG


def test_stage_validation_without_gpu():
    lib = V.load_library()
    fake = ctypes.c_void_p(4096)
    # N not a multiple of 128, K not a multiple of 64, misaligned pointer, null pointer
    assert lib.vit_stage_linear(fake, fake, fake, 8, 100, 64, 0, fake, fake, None) == V.VIT_E_SHAPE
    assert lib.vit_stage_linear(fake, fake, fake, 8, 128, 60, 0, fake, fake, None) == V.VIT_E_SHAPE
    assert lib.vit_stage_linear(ctypes.c_void_p(4100), fake, fake, 8, 128, 64, 0, fake, fake, None) == V.VIT_E_INVALID_ARG
    assert lib.vit_stage_attention(None, 1, 8, 1, fake, fake, None) == V.VIT_E_INVALID_ARG
    assert lib.vit_stage_attention(fake, 1, 0, 1, fake, fake, None) == V.VIT_E_SHAPE
    assert lib.vit_workspace_size(None, 1, None) == V.VIT_E_INVALID_ARG
    assert lib.vit_status_str(V.VIT_E_DEVICE_TIMEOUT) == b"device pipeline wait timed out"
