"""The C-ABI library builds for sm_100a, loads, and exports every entry point that
include/moe.h declares (no compute calls: this runs without a GPU)."""
import ctypes
import os
import re

import torch

from block_scaled_moe_sigmoid_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_plan_create", "moe_route", "moe_forward", "moe_quant_mxfp8", "moe_permute"):
        assert required in names


def test_library_exports_every_declared_symbol():
    path = build.build()
    L = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) == set(api.SIGNATURES)


def test_host_side_argument_checks_without_gpu():
    L = api.lib()
    h = ctypes.c_void_p()
    # bad shapes are rejected before anything touches a device
    assert L.moe_plan_create(16, 100, 8, 2, 128, 0, 0, 0, 0, ctypes.byref(h)) == 2
    assert L.moe_plan_create(16, 128, 8, 33, 128, 0, 0, 0, 0, ctypes.byref(h)) == 2
    assert L.moe_plan_create(16, 128, 8, 9, 128, 0, 0, 0, 0, ctypes.byref(h)) == 2
    assert L.moe_plan_create(-1, 128, 8, 2, 128, 0, 0, 0, 0, ctypes.byref(h)) == 1
    assert L.moe_plan_create(16, 128, 8, 2, 128, 0, 2, 0, 0, ctypes.byref(h)) == 1   # unknown act
    assert L.moe_plan_create(16, 128, 8, 2, 128, 0, 0, 2, 0, ctypes.byref(h)) == 1   # unknown bias mode
    assert L.moe_plan_create(16, 128, 8, 2, 128, 0, 0, 0, 2, ctypes.byref(h)) == 1   # unknown flag bit
    assert L.moe_plan_create(16, 128, 8, 2, 128, 0, 0, 0, 1, ctypes.byref(h)) == 0   # static router
    assert L.moe_plan_destroy(h) == 0
    # both activations and both bias modes are accepted (host-side plan only)
    for act, mode in ((1, 0), (0, 1), (1, 1)):
        assert L.moe_plan_create(16, 128, 8, 2, 128, 0, act, mode, 0, ctypes.byref(h)) == 0
        assert L.moe_plan_destroy(h) == 0
    # latent option: shape checks on a host-only plan (no workspace attached yet)
    assert L.moe_plan_create(16, 256, 8, 2, 128, 0, 0, 0, 0, ctypes.byref(h)) == 0
    assert L.moe_plan_set_latent(h, 100, ctypes.c_float(1e-5)) == 2     # not a multiple of 128
    assert L.moe_plan_set_latent(h, 384, ctypes.c_float(1e-5)) == 1     # wider than d
    assert L.moe_plan_set_latent(h, 128, ctypes.c_float(0.0)) == 1      # eps must be > 0
    n0 = ctypes.c_size_t()
    assert L.moe_plan_workspace_bytes(h, ctypes.byref(n0)) == 0
    assert L.moe_plan_set_latent(h, 128, ctypes.c_float(1e-5)) == 0
    n1 = ctypes.c_size_t()
    assert L.moe_plan_workspace_bytes(h, ctypes.byref(n1)) == 0
    assert n1.value > n0.value                                          # latent buffers added
    v = ctypes.c_int()
    for opt in (0, 1, 2, 3, 4, 5):
        assert L.moe_plan_get_option(h, opt, ctypes.byref(v)) == 0
    assert L.moe_plan_get_option(h, 99, ctypes.byref(v)) == 1
    assert L.moe_plan_set_option(h, 3, 1) == 1                          # read-only option
    for tile_n in (0, 32, 128, 160, 176):                               # the tile configurations
        assert L.moe_plan_set_option(h, 2, tile_n) == 0
    for tile_n in (-1, 16, 64, 96, 192, 256):
        assert L.moe_plan_set_option(h, 2, tile_n) == 1
    assert L.moe_plan_set_option(h, 0, 65) == 1                         # prefetch distance <= 64
    assert L.moe_plan_set_option(h, 0, 8) == 0 and L.moe_plan_set_option(h, 0, 0) == 0
    assert L.moe_plan_destroy(h) == 0
    assert L.moe_quant_mxfp8(None, 4, 33, None, None, None) == 2
    assert L.moe_status_string(3) == b"misaligned pointer"
    sizes = api.moe_expert_bytes(7168, 3072, 896)
    # 896 experts x 3 matrices x 7168 x 3072 x (0.5 + 1/32) bytes
    assert sum(sizes) == 896 * 3 * 7168 * 3072 * 17 // 32


def test_workspace_size_grows_with_tokens():
    L = api.lib()
    h1, h2 = ctypes.c_void_p(), ctypes.c_void_p()
    assert L.moe_plan_create(64, 7168, 896, 16, 3072, 3072, 0, 0, 0, ctypes.byref(h1)) == 0
    assert L.moe_plan_create(8192, 7168, 896, 16, 3072, 3072, 0, 0, 0, ctypes.byref(h2)) == 0
    n1, n2 = ctypes.c_size_t(), ctypes.c_size_t()
    L.moe_plan_workspace_bytes(h1, ctypes.byref(n1))
    L.moe_plan_workspace_bytes(h2, ctypes.byref(n2))
    assert 0 < n1.value < n2.value < 8 << 30
    L.moe_plan_destroy(h1)
    L.moe_plan_destroy(h2)


def test_missing_library_fails_loudly():
    """Without the compiled library there is no fallback: the binding raises."""
    import subprocess
    import sys
    code = ("import block_scaled_moe_sigmoid_b200.api as a\n"
            "a.LIB_PATH = '/nonexistent/libmoe_sm100.so'\n"
            "a._lib = None\n"
            "try:\n"
            "    a.lib()\n"
            "except RuntimeError as e:\n"
            "    print('raised', 'missing' in str(e))\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120,
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    assert r.returncode == 0 and r.stdout.strip() == "raised True", (r.stdout, r.stderr[-500:])


def test_synthetic_draws_are_reproducible_and_independent():
    from block_scaled_moe_sigmoid_b200 import synth
    wl = synth.custom(seed=5, T=16, d=128, E=4, k=2, I=128, I_shared=128, d_latent=128)
    a = synth.draw_expert(wl, 1)
    b = synth.draw_expert(wl, 1)
    c = synth.draw_expert(wl, 2)
    assert all(torch.equal(u, v) for u, v in zip(a, b))
    assert not torch.equal(a[0], c[0])
    assert not torch.equal(a[0], a[1])            # gate and up come from separate streams
    assert torch.equal(synth.draw_x(wl), synth.draw_x(wl))
    lat = synth.draw_latent(wl)
    assert lat[0].shape == (128, 128) and lat[1].dtype == torch.float32 and lat[2].shape == (128, 128)
    assert synth.draw_latent(synth.custom(seed=5)) is None
