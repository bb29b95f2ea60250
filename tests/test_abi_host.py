"""Host-side checks of the C-ABI library: it loads, exports every declared
symbol, rejects bad arguments before touching the GPU, and builds a segment
table whose tiles cover every W element exactly once.  No GPU needed."""
import ctypes
import os
import re

import numpy as np
import pytest

from weight_merge_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_merge_b200 import build
    build.build()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "adafuse.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(adafuse_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 10
    L = ctypes.CDLL(B.library_path())
    for s in syms:
        assert hasattr(L, s), s


def test_tile_size_and_strerror():
    assert B.adafuse_tile_size() == 128
    assert B.adafuse_strerror(0) == "ok"
    assert "invalid" in B.adafuse_strerror(B.ADAFUSE_ERR_INVALID_ARG)
    assert B.adafuse_last_error() == ""


def _desc(shapes, n_layers, E=4, r=8, alpha=16.0, ptr=16):
    ts = []
    for l in range(n_layers):
        for k, (o, i) in enumerate(shapes):
            ts.append((f"t{k}", o, i, ptr, ptr, ptr))
    return B.make_desc(n_layers, len(shapes), E, r, alpha, ts)


@pytest.mark.parametrize("shapes,L", [
    ([(256, 256), (256, 256)], 2),
    ([(4096, 4096), (11008, 4096), (4096, 11008)], 2),
    ([(200, 136), (8, 8), (1024, 4096), (136, 264)], 3),
])
def test_segment_table_covers_each_element_once(shapes, L):
    d = _desc(shapes, L)
    tab = B.adafuse_segment_table(d)
    T = B.adafuse_tile_size()
    # layer-major, then target, then row / col tile
    keys = [tuple(x) for x in tab]
    assert keys == sorted(keys)
    for l in range(L):
        for k, (o, i) in enumerate(shapes):
            sel = tab[(tab[:, 0] == l) & (tab[:, 1] == k)]
            assert len(sel) == -(-o // T) * -(-i // T)
            cover = np.zeros((o, i), dtype=np.int32)
            for _, _, r0, c0 in sel:
                assert r0 % T == 0 and c0 % T == 0 and r0 < o and c0 < i
                cover[r0:r0 + T, c0:c0 + T] += 1
            assert cover.min() == 1 and cover.max() == 1


@pytest.mark.parametrize("bad,code", [
    (dict(shapes=[(100, 64)]), B.ADAFUSE_ERR_UNSUPPORTED_SHAPE),
    (dict(shapes=[(64, 60)]), B.ADAFUSE_ERR_UNSUPPORTED_SHAPE),
    (dict(r=0), B.ADAFUSE_ERR_UNSUPPORTED_SHAPE),
    (dict(r=65), B.ADAFUSE_ERR_UNSUPPORTED_SHAPE),
    (dict(E=0), B.ADAFUSE_ERR_UNSUPPORTED_SHAPE),
    (dict(E=65), B.ADAFUSE_ERR_UNSUPPORTED_SHAPE),
    (dict(alpha=float("nan")), B.ADAFUSE_ERR_INVALID_ARG),
    (dict(shapes=[(0, 64)]), B.ADAFUSE_ERR_INVALID_ARG),
])
def test_bad_descriptors_rejected_on_host(bad, code):
    kw = dict(shapes=[(64, 64)], L=1, E=4, r=8, alpha=16.0)
    kw.update(bad)
    d = _desc(kw["shapes"], kw["L"], kw["E"], kw["r"], kw["alpha"])
    n = ctypes.c_int64()
    assert B.lib().adafuse_segment_table(ctypes.byref(d), None, 0, ctypes.byref(n)) == code
    h = ctypes.c_void_p()
    assert B.lib().adafuse_create(ctypes.byref(h), ctypes.byref(d), 0) == code
    assert h.value is None


def test_create_rejects_null_and_misaligned_pointers():
    h = ctypes.c_void_p()
    assert B.lib().adafuse_create(ctypes.byref(h), None, 0) == B.ADAFUSE_ERR_INVALID_ARG
    d = _desc([(64, 64)], 1, ptr=0)
    assert B.lib().adafuse_create(ctypes.byref(h), ctypes.byref(d), 0) == B.ADAFUSE_ERR_INVALID_ARG
    d = _desc([(64, 64)], 1, ptr=24)
    assert B.lib().adafuse_create(ctypes.byref(h), ctypes.byref(d), 0) == B.ADAFUSE_ERR_INVALID_ARG


def test_calls_on_null_context_are_invalid():
    L = B.lib()
    assert L.adafuse_switch(None, None, None, None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_switch_batch_layers(None, 0, 1, None, None, None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_pregate(None, None, 1, 8, None, None, None) == B.ADAFUSE_ERR_INVALID_ARG
    st = ctypes.c_int32()
    assert L.adafuse_get_device_status(None, None, ctypes.byref(st)) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_pregate_topk(None, None, 1, 8, None, 2, None, None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_switch_topk(None, None, None, None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_switch_topk_layers(None, 0, 1, None, None, None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_rebase_topk(None, None, None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_set_tile_schedule(None, B.ADAFUSE_SCHEDULE_DYNAMIC) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_set_tile_schedule(None, B.ADAFUSE_SCHEDULE_AUTO) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_refresh_adapters(None, None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_get_topk_switch_kernel(None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_get_tensor_map_layout(None) == B.ADAFUSE_ERR_INVALID_ARG
    assert L.adafuse_destroy(None) == B.ADAFUSE_OK


def test_segment_table_capacity_checked():
    d = _desc([(256, 256)], 1)
    n = ctypes.c_int64()
    buf = (ctypes.c_int32 * 8)()
    assert B.lib().adafuse_segment_table(ctypes.byref(d), buf, 2, ctypes.byref(n)) == B.ADAFUSE_ERR_INVALID_ARG
    assert n.value == 4


def test_header_is_plain_c_and_links(tmp_path):
    """include/adafuse.h compiles as C99 with warnings as errors, and a C
    program that takes the address of every declared entry point links
    against the library and runs its host-only calls (no GPU work)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    syms = declared_symbols()
    lib = B.library_path()
    src = tmp_path / "abi_check.c"
    src.write_text(
        '#include <stdio.h>\n#include <string.h>\n#include "adafuse.h"\n'
        "int main(void) {\n"
        "    const void* fns[] = {\n" + "".join(f"        (const void*)&{s},\n" for s in syms) +
        "    };\n"
        "    adafuse_ctx* ctx = 0;\n"
        "    int64_t n = -1;\n"
        "    adafuse_target tg;\n"
        "    adafuse_desc d;\n"
        "    memset(&tg, 0, sizeof tg);\n"
        "    memset(&d, 0, sizeof d);\n"
        "    tg.out = 256; tg.in = 384;\n"
        "    d.n_layers = 1; d.n_targets = 1; d.n_experts = 2; d.rank = 8; d.alpha = 16.0f;\n"
        "    d.targets = &tg;\n"
        "    if (fns[0] == 0) return 1;\n"
        "    if (adafuse_tile_size() != 128) return 2;\n"
        "    if (adafuse_create(&ctx, 0, 0) != ADAFUSE_ERR_INVALID_ARG) return 3;\n"
        "    if (adafuse_segment_table(&d, 0, 0, &n) != ADAFUSE_OK || n != 6) return 4;\n"
        "    printf(\"%s\\n\", adafuse_strerror(ADAFUSE_ERR_INVALID_ARG));\n"
        "    return 0;\n"
        "}\n")
    exe = tmp_path / "abi_check"
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), lib, "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip()
