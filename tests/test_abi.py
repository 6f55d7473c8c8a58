"""Host-side tests of the C ABI: the library loads, exports what include/gdn.h
declares, and rejects bad arguments before launching anything.

No GPU is touched: every call here returns from the host-side checks (or is
an empty no-op) before any CUDA call.
"""
import ctypes
import os
import re

import pytest

from gated_deltanet_chunk_02_b200 import build as B
from gated_deltanet_chunk_02_b200 import gdn

HEADER = os.path.join(B.ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return gdn.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_A-Z]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["gdn_build_A", "gdn_invert_neumann", "gdn_invert_fwdsub", "gdn_wy",
              "gdn_invert_neumann_i8", "gdn_chunk_wy_fused", "gdn_forward",
              "gdn_get_status", "gdn_last_error"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert sorted(declared_functions()) == sorted(gdn.EXPORTS + [
        n for n in declared_functions() if n not in gdn.EXPORTS])


FAKE = 0x10000          # aligned, never dereferenced: every call below fails its checks first
MISALIGNED = 0x10008


def sh(B=1, H=1, T=256, k=64, d=128):
    return gdn.GdnShape(B, H, T, k, d)


def P(x):
    return ctypes.c_void_p(x)


def last(lib):
    return lib.gdn_last_error().decode()


def test_bad_chunk_size(lib):
    rc = lib.gdn_build_A(P(FAKE), P(FAKE), P(FAKE), P(FAKE), sh(k=48), 0, None)
    assert rc == gdn.GDN_ERR_ARG and "chunk size" in last(lib)


def test_T_not_multiple_of_k(lib):
    rc = lib.gdn_invert_fwdsub(P(FAKE), P(FAKE), sh(T=100), None)
    assert rc == gdn.GDN_ERR_ARG and "multiple" in last(lib)


def test_unsupported_head_dim(lib):
    rc = lib.gdn_invert_fwdsub(P(FAKE), P(FAKE), sh(d=64), None)
    assert rc == gdn.GDN_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers(lib):
    rc = lib.gdn_invert_fwdsub(None, P(FAKE), sh(), None)
    assert rc == gdn.GDN_ERR_ARG and "A is NULL" in last(lib)
    rc = lib.gdn_invert_fwdsub(P(FAKE), P(MISALIGNED), sh(), None)
    assert rc == gdn.GDN_ERR_ALIGN and "T is not 16-byte aligned" in last(lib)
    rc = lib.gdn_wy(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(MISALIGNED), P(FAKE), P(FAKE), sh(), 1,
                    None)
    assert rc == gdn.GDN_ERR_ALIGN and "g is not" in last(lib)


@pytest.mark.parametrize("N,mask,S", [(0, 1, 0), (64, 1, 0), (3, 2, 0), (3, 1, -1), (3, 1, 65)])
def test_neumann_parameter_ranges(lib, N, mask, S):
    rc = lib.gdn_invert_neumann(P(FAKE), P(FAKE), sh(), N, mask, S, 0, None)
    assert rc == gdn.GDN_ERR_ARG
    rc = lib.gdn_chunk_wy_fused(P(FAKE), P(FAKE), P(FAKE), P(FAKE), N, mask, S, 0, P(FAKE),
                                P(FAKE), None, sh(), 1, None)
    assert rc == gdn.GDN_ERR_ARG


def test_wait_expiry_hook_arguments(lib):
    """The test hook of the bounded waits checks its arguments (valid ones
    are left for the GPU test: arming here would only be consumed by a launch)."""
    f = lib.gdn_debug_arm_wait_expiry
    assert f(-1, 0, ctypes.c_double(5.0)) == gdn.GDN_ERR_ARG and "negative" in last(lib)
    assert f(0, 2, ctypes.c_double(5.0)) == gdn.GDN_ERR_ARG
    assert f(0, 0, ctypes.c_double(0.0)) == gdn.GDN_ERR_ARG
    assert f(0, 1, ctypes.c_double(2500.0)) == gdn.GDN_ERR_ARG


def test_int8_limits(lib):
    assert lib.gdn_invert_neumann_i8(P(FAKE), P(FAKE), 3, 1, None, None, None, sh(k=128),
                                     None) == gdn.GDN_ERR_UNSUPPORTED
    assert lib.gdn_invert_neumann_i8(P(FAKE), P(FAKE), 9, 1, None, None, None, sh(),
                                     None) == gdn.GDN_ERR_ARG
    assert lib.gdn_invert_neumann_i8(P(FAKE), P(FAKE), 3, 1, P(MISALIGNED), None, None, sh(),
                                     None) == gdn.GDN_ERR_ALIGN


def test_float32_chain_limit_and_bad_enums(lib):
    assert lib.gdn_invert_neumann(P(FAKE), P(FAKE), sh(T=512, k=256), 3, 1, 0, 0,
                                  None) == gdn.GDN_ERR_UNSUPPORTED
    assert lib.gdn_invert_neumann(P(FAKE), P(FAKE), sh(), 3, 1, 0, 7, None) == gdn.GDN_ERR_ARG
    assert lib.gdn_build_A(P(FAKE), P(FAKE), P(FAKE), P(FAKE), sh(), 5, None) == gdn.GDN_ERR_ARG


def test_k256_chain_limits(lib):
    # N runs up to k - 1
    assert lib.gdn_invert_neumann(P(FAKE), P(FAKE), sh(T=512, k=256), 256, 1, 0, 1,
                                  None) == gdn.GDN_ERR_ARG
    # the fused and WY kernels stop at k=128
    assert lib.gdn_chunk_wy_fused(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 3, 1, 0, 0, P(FAKE), P(FAKE),
                                  None, sh(T=512, k=256), 1, None) == gdn.GDN_ERR_UNSUPPORTED


def test_empty_inputs_are_noops(lib):
    n0 = lib.gdn_launch_count()
    for s in (sh(B=0), sh(H=0), sh(T=0)):
        assert lib.gdn_build_A(None, None, None, None, s, 1, None) == gdn.GDN_OK
        assert lib.gdn_invert_fwdsub(None, None, s, None) == gdn.GDN_OK
        assert lib.gdn_chunk_wy_fused(None, None, None, None, 3, 1, 8, 0, None, None, None, s, 1,
                                      None) == gdn.GDN_OK
    assert lib.gdn_launch_count() == n0


def test_int8_residual_limits(lib):
    assert lib.gdn_invert_neumann_i8_residual(P(FAKE), P(FAKE), 3, 1, 0, sh(), None) == gdn.GDN_ERR_ARG
    assert lib.gdn_invert_neumann_i8_residual(P(FAKE), P(FAKE), 3, 1, 8, sh(k=128),
                                              None) == gdn.GDN_ERR_UNSUPPORTED
    assert lib.gdn_invert_neumann_i8_residual(None, None, 3, 1, 8, sh(B=0), None) == gdn.GDN_OK


def test_int16_limits(lib):
    assert lib.gdn_invert_neumann_i16(P(FAKE), P(FAKE), 3, 1, None, None, None, sh(k=128),
                                      None) == gdn.GDN_ERR_UNSUPPORTED
    assert lib.gdn_invert_neumann_i16(P(FAKE), P(FAKE), 9, 1, None, None, None, sh(),
                                      None) == gdn.GDN_ERR_ARG
    assert lib.gdn_invert_neumann_i16(P(FAKE), P(FAKE), 3, 1, None, P(MISALIGNED), None, sh(),
                                      None) == gdn.GDN_ERR_ALIGN
    assert lib.gdn_invert_neumann_i16(None, None, 3, 1, None, None, None, sh(B=0),
                                      None) == gdn.GDN_OK


def test_int16_residual_limits(lib):
    f = lib.gdn_invert_neumann_i16_residual
    assert f(P(FAKE), P(FAKE), 3, 1, 0, sh(), None) == gdn.GDN_ERR_ARG           # S < 1
    assert f(P(FAKE), P(FAKE), 3, 1, 65, sh(), None) == gdn.GDN_ERR_ARG          # S > 64
    assert f(P(FAKE), P(FAKE), 9, 1, 8, sh(), None) == gdn.GDN_ERR_ARG           # N > 8
    assert f(P(FAKE), P(FAKE), 3, 2, 8, sh(), None) == gdn.GDN_ERR_ARG           # mask
    assert f(P(FAKE), P(FAKE), 3, 1, 8, sh(k=128), None) == gdn.GDN_ERR_UNSUPPORTED
    assert f(P(MISALIGNED), P(FAKE), 3, 1, 8, sh(), None) == gdn.GDN_ERR_ALIGN
    assert f(None, None, 3, 1, 8, sh(B=0), None) == gdn.GDN_OK


def test_prologue_limits(lib):
    args = [P(FAKE)] * 4
    outs = [P(FAKE), P(FAKE), None, None, None]
    assert lib.gdn_chunk_wy_fused_raw(*args, 3, 1, 8, 0, *outs, sh(), 0, None) == \
        gdn.GDN_ERR_UNSUPPORTED                                  # float32 data
    assert lib.gdn_chunk_wy_fused_raw(*args, 3, 1, 8, 0, *outs, sh(T=512, k=256), 1, None) == \
        gdn.GDN_ERR_UNSUPPORTED
    bad = [P(FAKE), P(FAKE), None, P(MISALIGNED), None]
    assert lib.gdn_chunk_wy_fused_raw(*args, 3, 1, 8, 0, *bad, sh(), 1, None) == gdn.GDN_ERR_ALIGN
    assert lib.gdn_chunk_wy_fused_raw(*[None] * 4, 3, 1, 8, 0, *[None] * 5, sh(B=0), 1,
                                      None) == gdn.GDN_OK


def test_blocked_limits(lib):
    assert lib.gdn_invert_blocked(P(FAKE), P(FAKE), sh(k=128), None) == gdn.GDN_ERR_UNSUPPORTED
    assert lib.gdn_invert_blocked(P(FAKE), P(MISALIGNED), sh(), None) == gdn.GDN_ERR_ALIGN
    assert lib.gdn_invert_blocked(None, None, sh(B=0), None) == gdn.GDN_OK


def test_newton_limits(lib):
    assert lib.gdn_invert_newton(P(FAKE), P(FAKE), sh(), 3, 1, 7, None) == gdn.GDN_ERR_ARG
    assert lib.gdn_invert_newton(P(FAKE), P(FAKE), sh(), 0, 1, 2, None) == gdn.GDN_ERR_ARG
    assert lib.gdn_invert_newton(P(FAKE), P(FAKE), sh(T=512, k=256), 3, 1, 2,
                                 None) == gdn.GDN_ERR_UNSUPPORTED
    assert lib.gdn_invert_newton(P(FAKE), P(MISALIGNED), sh(), 3, 1, 2, None) == gdn.GDN_ERR_ALIGN
    assert lib.gdn_invert_newton(None, None, sh(B=0), 3, 1, 2, None) == gdn.GDN_OK


def test_decode_argument_checks(lib):
    n0 = lib.gdn_launch_count()
    args = [P(FAKE)] * 7
    # Hv not a multiple of Hk, head dim, bad dtype, misaligned state, empty
    assert lib.gdn_decode(*args, 1, 3, 4, 1, 128, 1, None) == gdn.GDN_ERR_ARG
    assert lib.gdn_decode(*args, 1, 2, 4, 1, 64, 1, None) == gdn.GDN_ERR_UNSUPPORTED
    assert lib.gdn_decode(*args, 1, 2, 4, 1, 128, 9, None) == gdn.GDN_ERR_ARG
    bad = args[:5] + [P(MISALIGNED), P(FAKE)]
    assert lib.gdn_decode(*bad, 1, 2, 4, 1, 128, 1, None) == gdn.GDN_ERR_ALIGN
    assert lib.gdn_decode(*[None] * 7, 1, 2, 4, 0, 128, 1, None) == gdn.GDN_OK
    assert lib.gdn_decode(*[None] * 7, 0, 2, 4, 1, 128, 1, None) == gdn.GDN_OK
    assert lib.gdn_decode(*[None] * 7, 1, 2, 4, 1, 128, 1, None) == gdn.GDN_ERR_ARG
    assert lib.gdn_launch_count() == n0


def test_workspace_size(lib):
    s = sh(B=2, H=3, T=512, k=64)
    nc = 2 * 3 * 8
    # W_g and U (bf16) plus A and T (fp32) for every chunk
    assert lib.gdn_forward_workspace_bytes(s, 1) == 2 * nc * 64 * 128 * 2 + 2 * nc * 64 * 64 * 4
    assert lib.gdn_forward_workspace_bytes(sh(k=48), 1) == -1
