"""Host-only checks of the C-ABI library: it loads, exports every symbol include/soup.h
declares, and its pure host calls (layout, sizes, validation, codebook) behave.  No kernel
runs here."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from layer_streamed_nf4_lut_b200 import _lib, model as M
from oracle import nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "soup.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(soup_[a-z0-9_]+)\s*\(", hdr)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 25
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_binding_covers_header():
    names = set(declared_symbols())
    bound = set(_lib.SIGNATURES) | set(_lib.STRING_FUNCS)
    assert names == bound, names ^ bound


def test_codebook_bitwise_equals_oracle():
    # the library derives its levels in C++ (bisection + Newton on erfc); the oracle with scipy
    assert np.array_equal(M.codebook().view(np.uint32), nf4.codebook().view(np.uint32))


def test_blob_layout_matches_format_sizes():
    for cfg in (synth.TINY, synth.L8B, synth.L70B):
        total = M.blob_bytes(cfg)
        algo = 0
        for p, name in enumerate(synth.PROJ_NAMES):
            o, i = synth.proj_shape(cfg, name)
            want = nf4.blob_segment_bytes(o * i)
            for part, key in enumerate(("codes", "q8", "scales", "mean")):
                off, sz = M.blob_part(cfg, p, part)
                assert sz == want[key] and off % 256 == 0
                algo += sz
        for g in (7, 8):
            off, sz = M.blob_part(cfg, g, 0)
            assert sz == 2 * cfg["hidden"] and off % 256 == 0
            algo += sz
        assert algo == nf4.layer_stream_bytes([np.prod(synth.proj_shape(cfg, p)) for p in synth.PROJ_NAMES],
                                              cfg["hidden"])
        assert algo <= total < algo + 256 * 30
    assert abs(M.blob_bytes(synth.L8B) / 1e6 - 112.53) < 0.01
    assert abs(M.blob_bytes(synth.L70B) / 1e6 - 441.43) < 0.05


def test_lora_layout_contiguous_and_complete():
    cfg = synth.TINY
    n = M.lora_numel(cfg)
    r = cfg["lora_r"]
    seen = np.zeros(n, dtype=np.int32)
    for layer in range(cfg["n_layers"]):
        for p, name in enumerate(synth.PROJ_NAMES):
            o, i = synth.proj_shape(cfg, name)
            offA, ra, ca = M.lora_offset(cfg, layer, p, 0)
            offB, rb, cb = M.lora_offset(cfg, layer, p, 1)
            assert (ra, ca) == (r, i) and (rb, cb) == (o, r)
            seen[offA:offA + ra * ca] += 1
            seen[offB:offB + rb * cb] += 1
    assert np.all(seen == 1)
    # stacked q|k|v A's and B's are contiguous (the kernels rely on it)
    a_q, _, _ = M.lora_offset(cfg, 0, 0, 0)
    a_k, _, _ = M.lora_offset(cfg, 0, 1, 0)
    assert a_k == a_q + r * cfg["hidden"]
    assert M.lora_numel(synth.L8B) == 167772160


@pytest.mark.parametrize("field,value,status", [("head_dim", 96, -7), ("n_heads", 5, -1), ("hidden", 250, -7),
                                                ("lora_r", 6, -7), ("n_layers", 0, -1)])
def test_config_validation(field, value, status):
    cfg = dict(synth.TINY)
    cfg[field] = value
    n = ctypes.c_size_t()
    st = _lib.lib.soup_layer_blob_bytes(ctypes.byref(M.make_config(cfg)), ctypes.byref(n))
    assert st == status


def test_stream_source_validation():
    n = ctypes.c_size_t()
    bad = M.make_config(synth.TINY)
    bad.stream_source = 7
    assert _lib.lib.soup_layer_blob_bytes(ctypes.byref(bad), ctypes.byref(n)) == -1
    nopath = M.make_config(synth.TINY, source="file")
    assert _lib.lib.soup_layer_blob_bytes(ctypes.byref(nopath), ctypes.byref(n)) == -1
    ok = M.make_config(synth.TINY, source="file", stack_path="/tmp/x.soup")
    assert _lib.lib.soup_layer_blob_bytes(ctypes.byref(ok), ctypes.byref(n)) == 0
    assert _lib.lib.soup_status_string(-8) == b"layer stack file I/O failed"


def test_streamed_needs_two_buffers():
    c = M.make_config(synth.TINY, mode="streamed", n_layer_buffers=1)
    h = ctypes.c_void_p()
    assert _lib.lib.soup_model_create(ctypes.byref(c), None, ctypes.byref(h)) == -1


def test_null_arguments_rejected():
    L = _lib.lib
    assert L.soup_model_destroy(None) == -1
    assert L.soup_set_lora_enabled(None, 1) == -1
    assert L.soup_step(None, 0, None, None, None) == -1
    assert L.soup_nf4_codebook(None) == -1
    assert L.soup_status_string(-5) == b"timed out"


def test_struct_layouts_match_the_c_compiler(tmp_path):
    """sizeof / offsetof of every public struct, as gcc lays them out from include/soup.h,
    against the ctypes mirrors the binding passes across the boundary."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    structs = {"soup_model_config": _lib.ModelConfig, "soup_allocator": _lib.Allocator, "soup_stats": _lib.Stats,
               "soup_profile_entry": _lib.ProfileEntry, "soup_batch": _lib.Batch,
               "soup_gemm_plan_info": _lib.GemmPlanInfo}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "soup.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'  printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for cname, cls in structs.items():
        assert got[(cname, "sizeof")] == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert got[(cname, fname)] == getattr(cls, fname).offset, (cname, fname)
