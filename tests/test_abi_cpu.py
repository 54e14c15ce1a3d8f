"""The C ABI without a GPU: the library loads, exports every declared
entry point, its host CG generator matches the oracle, and argument errors
are reported before any device work."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import cg as ocg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from equivariant_mlip_tensor_b200 import lib
    return lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "cgtp.h")).read()
    return sorted(set(re.findall(r"\b(cgtp_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n
    from equivariant_mlip_tensor_b200._lib import SIGNATURES
    assert sorted(SIGNATURES) == names


def test_host_cg_generator_matches_oracle():
    from equivariant_mlip_tensor_b200 import api
    for l1 in range(5):
        for l2 in range(5):
            for l3 in range(abs(l1 - l2), min(l1 + l2, 4) + 1):
                assert np.allclose(api.cg_block(l1, l2, l3), ocg.real_cg(l1, l2, l3), atol=1e-12, rtol=0)
    assert np.all(api.cg_block(1, 1, 3) == 0.0)  # outside the triangle: zero block


def test_status_strings_and_host_side_errors(L):
    assert L.cgtp_status_string(0) == b"CGTP_OK"
    assert L.cgtp_status_string(7) == b"CGTP_ERR_WORKSPACE"
    h = ctypes.c_void_p()
    assert L.cgtp_plan_create(1, 1, 1, 6, 0, ctypes.byref(h)) == 1      # mult not a multiple of 4
    assert L.cgtp_plan_create(-1, 1, 1, 8, 0, ctypes.byref(h)) == 1
    assert L.cgtp_plan_create(2, 3, 1, 8, 0, ctypes.byref(h)) == 2      # shape not compiled in
    assert L.cgtp_plan_create(2, 3, 2, 8, 3, ctypes.byref(h)) == 2      # not built for the fully connected mode
    assert L.cgtp_plan_create(1, 1, 1, 8, 9, ctypes.byref(h)) == 1      # unknown mode
    assert L.cgtp_plan_create(1, 1, 1, 8, 0, None) == 1
    assert L.cgtp_conv_forward(None, 1, 0, None, None, None, None, None, None, None) == 1
    assert L.cgtp_plan_set_checked(None, 1) == 1
    assert L.cgtp_plan_check(None, None) == 1
    assert L.cgtp_cg_block(5, 0, 5, None) == 1
    assert L.cgtp_supported(2, 4, 2, 0) == 1 and L.cgtp_supported(4, 4, 4, 0) == 0
    sz = ctypes.c_size_t()
    assert L.cgtp_conv_backward_workspace_size(None, 10, ctypes.byref(sz)) == 1
    bad = ctypes.c_void_p(0x1004)  # misaligned for float4 access
    assert L.cgtp_graph_build(None, 5, ctypes.c_float(0), ctypes.c_float(1.0), None, 0, None, None, None,
                              None, None, None, 0, None, None) == 1
    assert L.cgtp_forces(-1, 0, bad, bad, None, None, None, None) == 1


VARIANT_SHAPES = {(0, 0, 0), (1, 1, 1), (1, 2, 1), (2, 2, 2), (2, 4, 2), (3, 3, 3)}


def test_supported_shapes_follow_the_policy(L):
    """cgtp_supported and the build's shape lists agree with the documented
    policy: the channelwise convolution and the pair product for every
    interaction (lmax_in == lmax_out), embedding (lmax_in == 0) and read-out
    (lmax_out == 0) shape with lmax_in, lmax_out <= 3 and lmax_sh <= 4; the
    weight-structure variants for the shapes of the standard workloads."""
    from equivariant_mlip_tensor_b200 import build
    uvu_list = set()
    for li in range(6):
        for ls in range(6):
            for lo in range(6):
                uvu = li <= 3 and lo <= 3 and ls <= 4 and (li == lo or li == 0 or lo == 0)
                var = (li, ls, lo) in VARIANT_SHAPES
                if uvu:
                    uvu_list.add((li, ls, lo))
                assert L.cgtp_supported(li, ls, lo, 0) == int(uvu), (li, ls, lo)   # CONV_UVU
                assert L.cgtp_supported(li, ls, lo, 1) == int(uvu), (li, ls, lo)   # PAIR_UVU
                assert L.cgtp_supported(li, ls, lo, 2) == int(var), (li, ls, lo)   # CONV_UVU_SHARED
                assert L.cgtp_supported(li, ls, lo, 3) == int(var), (li, ls, lo)   # CONV_UVW
    assert L.cgtp_supported(2, 2, 2, 7) == 0
    assert set(build.shapes()) == uvu_list and len(uvu_list) == 50
    assert set(build.shapes("CGTP_VARIANT_CONFIGS")) == VARIANT_SHAPES
