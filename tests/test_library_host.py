"""CPU-only checks of the C-ABI library: it loads, exports every entry point
declared in include/tq.h, rejects bad arguments before touching CUDA, and its
host-side parameters (Pi, S, codebooks) equal the oracle's, which computes
them independently."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import turboquant_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_12_b200 import build
    build.build()
    from kv_cache_vector_12_b200 import tq as tqmod
    return tqmod


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(tq_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(tq):
    names = _declared_functions()
    assert "tq_create" in names and "tq_decode_attention" in names
    for n in names:
        assert hasattr(tq.lib, n), n


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("law", [o.LAW_GAUSSIAN, o.LAW_SPHERE])
@pytest.mark.parametrize("bits_k,bits_v,qjl,seed", [(3, 3, 0, 42), (2, 4, 1, 42), (4, 2, 1, 7), (3, 2, 0, 12345)])
def test_host_params_equal_oracle(tq, d, bits_k, bits_v, qjl, seed, law):
    lib_p = tq.host_params(d, bits_k, bits_v, qjl, seed, law=law)
    ref = o.Params(d, bits_k, bits_v, bool(qjl), seed, law)
    assert np.array_equal(lib_p["pi"].double().numpy(), ref.pi)
    assert np.array_equal(lib_p["centroids_k"].double().numpy(), ref.ck)
    assert np.array_equal(lib_p["thresholds_k"].double().numpy(), ref.tk)
    assert np.array_equal(lib_p["centroids_v"].double().numpy(), ref.cv)
    assert np.array_equal(lib_p["thresholds_v"].double().numpy(), ref.tv)
    if qjl:
        assert np.array_equal(lib_p["s"].double().numpy(), ref.s)


def test_cache_struct_layout_matches_header(tq, tmp_path):
    """The binding's tq_cache mirrors include/tq.h field for field: a C
    program compiled against the header prints sizeof and every offsetof."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = [f[0] for f in tq.tq_cache._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"tq.h\"\nint main(void) {\n"
                   + "".join(f'  printf("%zu\\n", offsetof(tq_cache, {f}));\n' for f in fields)
                   + '  printf("%zu\\n", sizeof(tq_cache));\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    # the header's CUDA-free part only: tq.h includes nothing from CUDA
    subprocess.run([cc, "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [getattr(tq.tq_cache, f).offset for f in fields] + [ctypes.sizeof(tq.tq_cache)]
    assert got == want


def test_invalid_arguments_fail_before_cuda(tq):
    lib = tq.lib
    f = ctypes.POINTER(ctypes.c_float)()
    assert lib.tq_host_params(128, 5, 3, 0, 1, f, f, f, f, f, f) == tq.TQ_ERR_INVALID
    assert b"bits" in lib.tq_last_error()
    assert lib.tq_host_params(128, 3, 3, 2, 1, f, f, f, f, f, f) == tq.TQ_ERR_INVALID
    assert lib.tq_host_params_ex(128, 3, 3, 0, 1, 2, f, f, f, f, f, f) == tq.TQ_ERR_INVALID
    assert b"law" in lib.tq_last_error()
    assert lib.tq_create_ex(None, 128, 3, 3, 0, 1, 1) == tq.TQ_ERR_INVALID
    h = ctypes.c_void_p()
    assert lib.tq_create(ctypes.byref(h), 96, 3, 3, 0, 1) == tq.TQ_ERR_UNSUPPORTED
    assert b"64, 128 or 256" in lib.tq_last_error()
    assert lib.tq_create(None, 128, 3, 3, 0, 1) == tq.TQ_ERR_INVALID
    assert lib.tq_quantize(None, None, None, None, None, None, 0, None) == tq.TQ_ERR_INVALID
    assert lib.tq_decode_attention(None, None, None, 0, 1, None, 1, 0.0, None, None, None, 0, None) == \
        tq.TQ_ERR_INVALID
    assert lib.tq_layout(None, None) == tq.TQ_ERR_INVALID
    assert lib.tq_workspace_bytes(None, 1, 1, 1) == 0
    lib.tq_destroy(None)


def test_binding_has_no_fallback_when_library_missing(tmp_path):
    """Importing the binding from a package copy without libtq.so must raise."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "kv_cache_vector_12_b200"
    pkg.mkdir()
    for fn in ("__init__.py", "tq.py"):
        shutil.copy(os.path.join(ROOT, "kv_cache_vector_12_b200", fn), pkg / fn)
    r = subprocess.run([sys.executable, "-c", "import kv_cache_vector_12_b200.tq"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libtq.so" in r.stderr
