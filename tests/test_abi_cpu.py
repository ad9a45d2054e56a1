"""The C ABI library builds, loads and exports every symbol include/dg.h declares (CPU only).

No compute call is made here: only host-side helpers that touch no device.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from discrete_diffusion_decoding_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("dg_canvas_init", "dg_denoise_step", "dg_stop_check", "dg_stub_hidden", "dg_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_binding_covers_the_header():
    from discrete_diffusion_decoding_b200 import _abi
    assert sorted(_abi.EXPORTS) == _declared()


def test_host_helpers_without_device(lib):
    from discrete_diffusion_decoding_b200 import _abi
    p = _abi.DgParams()
    lib.dg_params_default.argtypes = [ctypes.POINTER(_abi.DgParams), ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.dg_params_default(ctypes.byref(p), 16, 262144, 2816)
    assert (p.n_canvas, p.canvas_len, p.vocab, p.hidden, p.max_steps) == (16, 256, 262144, 2816, 48)
    assert abs(p.t_start - 0.8) < 1e-7 and abs(p.t_end - 0.4) < 1e-7
    assert abs(p.eb_bound - 0.1) < 1e-7 and abs(p.stop_thresh - 0.005) < 1e-9 and p.stability == 2
    lib.dg_temperature.argtypes = [ctypes.POINTER(_abi.DgParams), ctypes.c_int]
    lib.dg_temperature.restype = ctypes.c_float
    from oracle import stage
    for s in (1, 2, 17, 48):
        assert lib.dg_temperature(ctypes.byref(p), s) == stage.temperature(s, 48)
    lib.dg_status_string.restype = ctypes.c_char_p
    assert lib.dg_status_string(-4) == b"in-kernel wait timed out"


def test_sm100a_only_build():
    from discrete_diffusion_decoding_b200 import build
    src = open(build.__file__).read()
    assert "arch=compute_100a,code=sm_100a" in src


def test_last_sm_clock_argument_checks_without_device(lib):
    from discrete_diffusion_decoding_b200 import _abi
    p = _abi.DgParams()
    lib.dg_params_default(ctypes.byref(p), 1, 4096, 512)
    lib.dg_last_sm_clock.argtypes = [ctypes.POINTER(_abi.DgParams), ctypes.c_void_p, ctypes.c_size_t,
                                     ctypes.POINTER(ctypes.c_float), ctypes.c_void_p]
    lib.dg_last_sm_clock.restype = ctypes.c_int
    mhz = ctypes.c_float()
    assert lib.dg_last_sm_clock(ctypes.byref(p), None, 1 << 20, ctypes.byref(mhz), None) == _abi.DG_EINVAL
    assert lib.dg_last_sm_clock(ctypes.byref(p), 1 << 20, 1 << 20, None, None) == _abi.DG_EINVAL


def test_defaults_match_the_pages_settings_table(lib):
    """dg_params_default and the oracle's defaults carry the settings the pages print
    (tests/golden/sampler_settings.txt)."""
    import inspect

    from discrete_diffusion_decoding_b200 import _abi
    from oracle import decode, stage
    want = {}
    for line in open(os.path.join(ROOT, "tests", "golden", "sampler_settings.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            want[k] = float(v)
    p = _abi.DgParams()
    lib.dg_params_default(ctypes.byref(p), 1, 4096, 128)
    for k, v in want.items():
        assert abs(getattr(p, k) - v) <= 1e-7 * max(1.0, v), k
    sig = inspect.signature(decode.decode_batch).parameters
    assert sig["max_steps"].default == want["max_steps"] and sig["t_start"].default == want["t_start"]
    assert sig["t_end"].default == want["t_end"] and sig["bound"].default == want["eb_bound"]
    assert sig["stop_thresh"].default == want["stop_thresh"] and sig["stability"].default == want["stability"]
    # the schedule's end points (the oracle returns T in float32, the precision the kernel takes)
    assert abs(stage.temperature(1, 48) - want["t_start"]) <= 1e-7
    assert abs(stage.temperature(48, 48) - want["t_end"]) <= 1e-7


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++17")])
def test_header_compiles_standalone(lang, std):
    """include/dg.h is a plain C header: it compiles on its own as C99 and as C++ with warnings on."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = f'#include "{HEADER}"\nint main(void) {{ dg_params p; (void)p; return 0; }}\n'
    out = subprocess.run([cc, f"-std={std}", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", lang, "-"],
                         input=src, capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr



def test_tile_head_argument_checks_without_device(lib):
    """dg_tile_head refuses bad shapes, null and overlapping pointers before touching a device."""
    lib.dg_tile_head.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_void_p]
    lib.dg_tile_head.restype = ctypes.c_int
    a, b = 1 << 20, 1 << 30                      # never dereferenced: every call below fails its checks
    for args in ((None, b, 256, 128, 0), (a, None, 256, 128, 0), (a, b, 200, 128, 0), (a, b, 256, 96, 0),
                 (a, b, 0, 128, 0), (a, b, 256, 128, 2), (a + 8, b, 256, 128, 0), (a, a + 4096, 256, 128, 0)):
        assert lib.dg_tile_head(*args, None) == -1, args
    from discrete_diffusion_decoding_b200 import _abi
    p = _abi.DgParams()
    lib.dg_params_default(ctypes.byref(p), 1, 4096, 512)
    assert p.head_layout == 0
