"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/la_api.h declares, and rejects bad arguments before it launches
anything.  No test here runs device code (fake pointers are only ever given
to calls that must refuse them during validation)."""
import ctypes
import os
import re

import pytest

from linear_attention_transformers_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "la_api.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LA_EXPORT\s+[\w\s\*]+?\b(la_\w+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for fn in ("la_forward", "la_backward", "la_decode_step", "la_workspace_size",
               "la_status_string", "la_get_device_error", "la_version"):
        assert fn in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.la_version() == 2


def test_status_strings(lib):
    for code in range(6):
        assert api.la_status_string(code)
    assert api.la_status_string(99) == "unknown status"


FAKE = 0x100000  # aligned, non-null, never dereferenced: every use below must fail validation


def fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, S=None, z=None, g=None, B=1, H=1, N=8, D=64, dt=1,
        causal=1, phi=0, ws=None, ws_bytes=0, pq=None, pk=None):
    return lib.la_forward(q, k, v, o, S, z, g, pq, pk, B, H, N, D, dt, causal, phi, ws, ws_bytes,
                          None)


def bwd(lib, p=FAKE, B=1, H=1, N=8, D=64, dt=1, causal=1, phi=0, ws=None, ws_bytes=0, dq=FAKE,
        o=None, g=None, pq=None, pk=None):
    return lib.la_backward(p, p, p, p, o, g, pq, pk, dq, p, p, B, H, N, D, dt, causal, phi, ws,
                           ws_bytes, None)


def test_rejects_bad_arguments_before_launch(lib):
    assert fwd(lib, q=None) == api.LA_ERR_INVALID_ARG
    assert fwd(lib, o=FAKE + 4) == api.LA_ERR_INVALID_ARG          # misaligned
    assert fwd(lib, D=48) == api.LA_ERR_UNSUPPORTED
    assert fwd(lib, D=0) == api.LA_ERR_INVALID_ARG
    assert fwd(lib, N=-1) == api.LA_ERR_INVALID_ARG
    assert fwd(lib, dt=7) == api.LA_ERR_INVALID_ARG
    assert fwd(lib, phi=9) == api.LA_ERR_INVALID_ARG
    assert fwd(lib, N=1 << 31) == api.LA_ERR_UNSUPPORTED
    assert fwd(lib, B=1 << 20, H=1 << 20, N=1 << 20) == api.LA_ERR_UNSUPPORTED
    assert bwd(lib, dq=None) == api.LA_ERR_INVALID_ARG
    assert bwd(lib, D=96) == api.LA_ERR_UNSUPPORTED
    assert fwd(lib, g=FAKE + 4) == api.LA_ERR_INVALID_ARG         # misaligned g
    # saved forward statistics go together: o without g is refused
    need = lib.la_workspace_size(api.LA_OP_BACKWARD, 1, 1, 8, 64, 1, api.LA_BF16)
    assert bwd(lib, o=FAKE, g=None, ws=FAKE, ws_bytes=need) == api.LA_ERR_INVALID_ARG
    # feature maps go together, and only with o and g
    assert fwd(lib, pq=FAKE) == api.LA_ERR_INVALID_ARG
    assert fwd(lib, pq=FAKE, pk=FAKE + 4) == api.LA_ERR_INVALID_ARG   # misaligned
    assert bwd(lib, pq=FAKE, pk=FAKE, ws=FAKE, ws_bytes=need) == api.LA_ERR_INVALID_ARG
    assert bwd(lib, o=FAKE, g=FAKE, pk=FAKE, ws=FAKE, ws_bytes=need) == api.LA_ERR_INVALID_ARG
    # grouped key/value heads: Hkv must divide H
    p = FAKE
    assert lib.la_forward_gqa(p, p, p, p, None, None, None, None, None, 1, 4, 3, 8, 64, 1, 1, 0,
                              None, 0, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_forward_gqa(p, p, p, p, None, None, None, None, None, 1, 4, 0, 8, 64, 1, 1, 0,
                              None, 0, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_decode_step_gqa(p, p, p, p, p, p, 2, 4, 3, 64, 1, 0, None) == \
        api.LA_ERR_INVALID_ARG
    # feature maps are per query head: not with shared key/value heads
    assert lib.la_forward_gqa(p, p, p, p, None, None, None, p, p, 1, 4, 2, 8, 64, 1, 1, 0,
                              None, 0, None) == api.LA_ERR_UNSUPPORTED
    assert lib.la_workspace_size_gqa(api.LA_OP_BACKWARD, 1, 4, 3, 8, 64, 1, 1) == 0
    assert lib.la_workspace_size_gqa(api.LA_OP_BACKWARD, 2, 4, 2, 1000, 64, 1, 1) > \
        lib.la_workspace_size(api.LA_OP_BACKWARD, 2, 4, 1000, 64, 1, 1)
    assert lib.la_selftest_wait_timeout(0, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_selftest_wait_timeout(2048, None) == api.LA_ERR_INVALID_ARG
    p = FAKE
    assert lib.la_decode_step(p, p, p, p, p, None, 2, 2, 64, 1, 0, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_decode_step(p, p, p, p, p, p, 2, 2, 40, 1, 0, None) == api.LA_ERR_UNSUPPORTED


def test_workspace_is_checked(lib):
    need = lib.la_workspace_size(api.LA_OP_BACKWARD, 2, 4, 1000, 64, 1, api.LA_BF16)
    assert need > 0
    assert bwd(lib, B=2, H=4, N=1000, ws=None, ws_bytes=0) == api.LA_ERR_WORKSPACE
    assert bwd(lib, B=2, H=4, N=1000, ws=FAKE, ws_bytes=need - 1) == api.LA_ERR_WORKSPACE
    assert bwd(lib, B=2, H=4, N=1000, ws=FAKE + 8, ws_bytes=need) == api.LA_ERR_INVALID_ARG
    # sizes that are rejected report no workspace
    assert lib.la_workspace_size(api.LA_OP_BACKWARD, 1, 1, 100, 48, 1, api.LA_BF16) == 0


def test_empty_sizes_launch_nothing(lib):
    # zero batch / heads / tokens: LA_OK with nothing launched (no final state asked)
    assert fwd(lib, B=0) == api.LA_OK
    assert fwd(lib, H=0) == api.LA_OK
    assert fwd(lib, N=0) == api.LA_OK
    assert bwd(lib, N=0) == api.LA_OK
    assert lib.la_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 64, 1, 0, None) == api.LA_OK


def test_decay_factors_are_validated_before_launch(lib):
    import ctypes
    p = FAKE

    def gam(*vals):
        return (ctypes.c_float * len(vals))(*vals)

    def fwd_decay(gamma, H=2, N=8, D=64):
        return lib.la_forward_decay(p, p, p, p, None, None, None, gamma, 1, H, N, D, 1, 0, None,
                                    0, None)

    assert fwd_decay(None) == api.LA_ERR_INVALID_ARG
    assert fwd_decay(gam(0.5, 1.5)) == api.LA_ERR_INVALID_ARG
    assert fwd_decay(gam(0.5, float("nan"))) == api.LA_ERR_INVALID_ARG
    assert fwd_decay(gam(-0.25, 0.5)) == api.LA_ERR_INVALID_ARG
    assert fwd_decay(gam(*([0.9] * 257)), H=257) == api.LA_ERR_UNSUPPORTED
    assert fwd_decay(gam(0.5, 0.9), D=40) == api.LA_ERR_UNSUPPORTED
    # valid factors, no tokens: nothing to launch
    assert fwd_decay(gam(0.5, 0.9), N=0) == api.LA_OK
    assert lib.la_backward_decay(p, p, p, p, None, None, p, p, p, gam(1.2, 0.5), 1, 2, 8, 64, 1,
                                 0, None, 0, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_decode_step_decay(p, p, p, p, p, p, gam(0.5, 2.0), 1, 2, 64, 1, 0, None) == \
        api.LA_ERR_INVALID_ARG
    assert lib.la_decode_step_decay(p, p, p, p, p, None, gam(0.5, 0.5), 1, 2, 64, 1, 0, None) == \
        api.LA_ERR_INVALID_ARG
    assert lib.la_workspace_size_decay(api.LA_OP_BACKWARD, 2, 4, 1000, 64, api.LA_BF16) >= \
        lib.la_workspace_size(api.LA_OP_BACKWARD, 2, 4, 1000, 64, 1, api.LA_BF16)


def test_favor_sizes_are_validated_before_launch(lib):
    p = FAKE
    # m = 256 or 32, float32, D = 32: not offered
    assert lib.la_favor_features(p, p, p, 1, 2, 8, 64, 256, api.LA_BF16, None) == \
        api.LA_ERR_UNSUPPORTED
    assert lib.la_favor_features(p, p, p, 1, 2, 8, 128, 32, api.LA_BF16, None) == \
        api.LA_ERR_UNSUPPORTED
    assert lib.la_favor_features(p, p, p, 1, 2, 8, 64, 64, api.LA_F32, None) == \
        api.LA_ERR_UNSUPPORTED
    assert lib.la_favor_features(p, p, p, 1, 2, 8, 32, 32, api.LA_BF16, None) == \
        api.LA_ERR_UNSUPPORTED
    assert lib.la_favor_features(p, p, p, -1, 2, 8, 64, 64, api.LA_BF16, None) == \
        api.LA_ERR_INVALID_ARG
    assert lib.la_favor_features(p, p, None, 1, 2, 8, 64, 64, api.LA_BF16, None) == \
        api.LA_ERR_INVALID_ARG
    assert lib.la_favor_features_backward(p, p, p, None, 1, 2, 8, 128, 128, api.LA_BF16,
                                          None) == api.LA_ERR_INVALID_ARG
    # nothing to do
    assert lib.la_favor_features(p, p, p, 1, 2, 0, 64, 64, api.LA_BF16, None) == api.LA_OK
    # the identity feature map is a valid enum
    assert lib.la_forward(p, p, p, None, None, None, None, None, None, 1, 1, 8, 64, api.LA_BF16,
                          1, 2, None, 0, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_forward(p, p, p, p, None, None, None, None, None, 1, 1, 8, 64, api.LA_BF16,
                          1, 3, None, 0, None) == api.LA_ERR_INVALID_ARG


def test_mv_calls_reject_bad_arguments_before_launch(lib):
    B, H, N = 1, 2, 100
    bf, f32 = api.LA_BF16, api.LA_F32

    def fwd(Dk=128, Dv=64, dt=bf, phi=0, ws=None, ws_bytes=0, q=FAKE):
        return lib.la_forward_mv(q, FAKE, FAKE, FAKE, None, B, H, N, Dk, Dv, dt, 1, phi, ws,
                                 ws_bytes, None)

    need = lib.la_workspace_size_mv(api.LA_OP_FORWARD, B, H, N, 128, 64, 1, bf)
    assert need >= 2 * B * H * N * 128 * 2  # widened v and o
    assert fwd(ws=FAKE, ws_bytes=need, q=None) == api.LA_ERR_INVALID_ARG
    assert fwd(Dk=96) == api.LA_ERR_UNSUPPORTED
    assert fwd(dt=f32) == api.LA_ERR_UNSUPPORTED
    assert fwd(Dk=64, Dv=128, phi=0) == api.LA_ERR_UNSUPPORTED      # zero features need identity
    assert fwd(ws=FAKE, ws_bytes=need - 256) == api.LA_ERR_WORKSPACE
    assert lib.la_workspace_size_mv(api.LA_OP_FORWARD, B, H, N, 128, 64, 1, f32) == 0
    need_b = lib.la_workspace_size_mv(api.LA_OP_BACKWARD, B, H, N, 64, 128, 1, bf)
    assert lib.la_backward_mv(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, B, H, N, 64,
                              128, bf, 1, 2, FAKE, need_b, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_backward_mv(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, B, H, N, 64,
                              128, bf, 1, 2, FAKE, need_b - 256, None) == api.LA_ERR_WORKSPACE
