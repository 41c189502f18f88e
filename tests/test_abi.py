"""The C-ABI library loads and exports every function include/lmoe.h declares (no GPU needed)."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lmoe.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lmoe_[a-z0-9_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def libmod():
    import __graft_entry__
    __graft_entry__._builder().build()
    import latentmoe_expert_layer_b200 as lm
    return lm


def test_header_declares_the_boundary():
    assert _declared() == sorted(["lmoe_create", "lmoe_load_weights", "lmoe_forward", "lmoe_forward_host",
                                  "lmoe_get_device_status", "lmoe_inspect", "lmoe_profile",
                                  "lmoe_profile_read", "lmoe_route_noalloc", "lmoe_export_nvfp4",
                                  "lmoe_selftest_wait_timeout", "lmoe_status_string",
                                  "lmoe_destroy", "lmoe_ep_dispatch", "lmoe_ep_experts", "lmoe_ep_combine"])


def test_library_exports_every_declared_symbol(libmod):
    out = subprocess.run(["nm", "-D", "--defined-only", libmod.library_path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (lmoe_[a-z0-9_]+)\b", out))
    missing = set(_declared()) - exported
    assert not missing, missing
    assert set(libmod.SYMBOLS) == set(_declared())


def test_status_strings(libmod):
    for code, name in libmod.STATUS.items():
        assert libmod.lib.lmoe_status_string(code).decode() == name


def test_create_rejects_bad_config_without_touching_a_gpu(libmod):
    import ctypes
    cfg = libmod._Config(256, 64, 16, 4, 128, 256, 64, 0, 0)
    h = ctypes.c_void_p()
    assert libmod.lib.lmoe_create(None, 0, ctypes.byref(h)) == 1
    bad = libmod._Config(250, 64, 16, 4, 128, 256, 64, 0, 0)        # d not a multiple of 64
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    bad = libmod._Config(256, 64, 16, 40, 128, 256, 64, 0, 0)       # K > 32
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    bad = libmod._Config(256, 64, 16, 4, 128, 256, 0, 0, 0)         # no tokens
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 1
    bad = libmod._Config(256, 64, 16, 4, 128, 256, 64, 1, 0, 2)     # unknown weight-scale rule
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 1
    bad = libmod._Config(256, 0, 16, 4, 128, 256, 64, 1, 0, 0)      # standard MoE (latent 0) in NVFP4
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    bad = libmod._Config(256, -64, 16, 4, 128, 256, 64, 0, 0, 0)    # negative latent
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 1
    assert libmod.lib.lmoe_forward(None, None, 0, None, None, None, None) == 1
    # expert parallelism: world above 8, rank outside the world, N not divisible, NVFP4, standard MoE
    bad = libmod._Config(256, 64, 16, 4, 128, 256, 64, 0, 0, 0, 9, 0)
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    bad = libmod._Config(256, 64, 16, 4, 128, 256, 64, 0, 0, 0, 2, 2)
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 1
    bad = libmod._Config(256, 64, 16, 4, 128, 256, 64, 0, 0, 0, 3, 0)
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    bad = libmod._Config(256, 128, 16, 4, 128, 256, 64, 1, 0, 0, 2, 0)
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    bad = libmod._Config(256, 0, 16, 4, 128, 256, 64, 0, 0, 0, 2, 0)
    assert libmod.lib.lmoe_create(ctypes.byref(bad), 0, ctypes.byref(h)) == 3
    assert libmod.lib.lmoe_ep_dispatch(None, None, 0, None, None, None, None, None, None, None, None) == 1
    del cfg


def test_no_device_is_reported(libmod):
    import ctypes
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = libmod._Config(256, 64, 16, 4, 128, 256, 64, 0, 0)
    h = ctypes.c_void_p()
    assert libmod.lib.lmoe_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == 9
