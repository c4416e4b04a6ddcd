"""The C ABI on the host: the library loads, exports every entry point that
include/psa.h declares, and rejects bad arguments before launching anything.
No GPU needed (no call here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest
import torch

import level_sparse_attention_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "psa.h")).read()
    return sorted(set(re.findall(r"^\S.*?\b(psa_\w+)\(", src, flags=re.M)))


def test_library_exports_every_declared_entry_point():
    L = P.lib()
    names = header_functions()
    assert set(names) == set(P.EXPORTED), names
    for n in names:
        assert hasattr(L, n), n


def test_debug_library_exports_the_same_entry_points():
    """libpsa_debug.so (PSA_DEBUG: device-side work-list bounds checks) is the
    same ABI; psa_debug_build tells the two apart."""
    D = P.debug_lib()
    for n in header_functions():
        assert hasattr(D, n), n
    assert D.psa_debug_build() == 1
    assert P.lib().psa_debug_build() == 0
    assert P.status_string(8).startswith("a work list")


def test_workspace_layout_matches_library():
    for w in [(1, 12, 12, 32760, 128, 128, torch.bfloat16), (1, 2, 2, 1024, 64, 64, torch.float32),
              (2, 28, 4, 16384, 128, 128, torch.bfloat16), (1, 3, 1, 77, 64, 128, torch.bfloat16)]:
        B, Hq, Hkv, N, d, qb, dt = w
        p = P.make_params(B, Hq, Hkv, N, d, q_blk=qb, dtype=dt)
        assert P.workspace_layout(p)["total"] == P.workspace_size(p)


@pytest.mark.parametrize("field,value", [
    ("d", 96), ("d", 0), ("Hkv", 3), ("q_blk", 32), ("kv_blk", 128), ("N", 0), ("B", -1),
    ("n_levels", 3), ("causal", 2), ("forced_prefix_tokens", -1), ("N", 64 * 8192 + 1)])
def test_invalid_params_give_zero_workspace(field, value):
    p = P.make_params(1, 10, 10, 4096, 128)
    setattr(p, field, value)
    assert P.workspace_size(p) == 0


@pytest.mark.parametrize("tau", [(0.5, 0.4, 0.9, 0.95), (0.0, 0.5, 0.9, 0.95),
                                 (0.5, 0.6, 0.9, 1.5), (float("nan"), 0.5, 0.9, 0.95)])
def test_bad_thresholds_rejected(tau):
    assert P.workspace_size(P.make_params(1, 2, 2, 1024, 64, tau=tau)) == 0


def test_bad_pool_rejected():
    p = P.make_params(1, 2, 2, 1024, 64)
    p.pool[2] = 3
    assert P.workspace_size(p) == 0


def _call_forward(p, q, k, v, o, ws, nbytes):
    return P.lib().psa_forward(ctypes.byref(p), q, k, v, o, None, None, ws, nbytes, None)


def test_argument_errors_before_any_launch():
    p = P.make_params(1, 2, 2, 1024, 64)
    need = P.workspace_size(p)
    A = ctypes.c_void_p(0x10000)            # aligned fake addresses: never dereferenced,
    B = ctypes.c_void_p(0x20000)            # every call below fails validation first
    mis = ctypes.c_void_p(0x10008)
    assert _call_forward(p, None, A, A, A, B, need) == 1            # NULL Q
    assert _call_forward(p, mis, A, A, A, B, need) == 3             # misaligned Q
    assert _call_forward(p, A, A, A, A, B, need - 1) == 4           # workspace too small
    assert _call_forward(p, A, A, A, A, ctypes.c_void_p(0x20010), need) == 3   # ws not 256-aligned
    assert _call_forward(p, A, A, A, A, None, need) == 1
    bad = P.make_params(1, 2, 2, 1024, 96)
    assert _call_forward(bad, A, A, A, A, B, need) == 2             # d = 96 unsupported
    assert P.lib().psa_build_pyramid(ctypes.byref(p), None, A, B, need, None) == 1
    mis4 = ctypes.c_void_p(0x10002)         # lse and block_mass need float (4-byte) alignment
    assert P.lib().psa_score_and_mask(ctypes.byref(p), A, B, need, None, mis4, None) == 3
    assert P.lib().psa_attention_fwd(ctypes.byref(p), A, A, A, B, need, None, A, mis4, None) == 3
    assert P.lib().psa_forward(ctypes.byref(p), A, A, A, A, mis4, None, B, need, None) == 3


def test_backward_argument_errors_before_any_launch():
    """psa_backward validates everything on the host before any launch: a
    NULL lse or scratch, a misaligned lse, scratch or tensor, scratch that is
    too small, and the forward workspace's own checks."""
    p = P.make_params(1, 4, 2, 1024, 64)
    need, bneed = P.workspace_size(p), P.backward_workspace_size(p)
    assert bneed > 0 and P.backward_workspace_size(P.make_params(1, 4, 2, 1024, 96)) == 0
    A, W, BW = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    f = lambda lse=A, bws=BW, bbytes=bneed, ws=W, wbytes=need, dq=A: P.lib().psa_backward(
        ctypes.byref(p), A, A, A, A, lse, A, None, ws, wbytes, bws, bbytes, dq, A, A, None)
    assert f(lse=None) == 1                                   # lse is required
    assert f(bws=None) == 1                                   # so is the scratch
    assert f(lse=ctypes.c_void_p(0x10002)) == 3               # lse: 4-byte alignment
    assert f(bws=ctypes.c_void_p(0x30010)) == 3               # scratch: 256-byte alignment
    assert f(bbytes=bneed - 1) == 4                           # scratch too small
    assert f(wbytes=need - 1) == 4                            # forward workspace too small
    assert f(dq=ctypes.c_void_p(0x10008)) == 3                # dQ: 16-byte alignment
    assert f(dq=None) == 1


def test_selftest_argument_errors_before_any_launch():
    p = P.make_params(1, 2, 2, 1024, 64)
    need = P.workspace_size(p)
    st = lambda ws, n, limit: P.lib().psa_selftest_wait_timeout(ctypes.byref(p), ws, n, limit, None)
    B = ctypes.c_void_p(0x20000)
    assert st(B, need, 0) == 1                                      # limit out of range
    assert st(B, need, 2_000_000_000) == 1
    assert st(None, need, 1000) == 1                                # NULL workspace
    assert st(ctypes.c_void_p(0x20010), need, 1000) == 3            # not 256-byte aligned
    assert st(B, need - 1, 1000) == 4                               # too small
    bad = P.make_params(1, 2, 2, 1024, 64)
    bad.N = 0
    assert P.lib().psa_selftest_wait_timeout(ctypes.byref(bad), B, need, 1000, None) == 1


def test_similarity_threshold_validated():
    """The cosine threshold: NaN or above 1 is rejected; -1 and below turn the
    constraint off and are valid."""
    for t in (-5.0, -1.0, 0.0, 0.95, 1.0):
        assert P.workspace_size(P.make_params(1, 2, 2, 1024, 64, sim_threshold=t)) > 0, t
    for t in (float("nan"), 1.0001, float("inf")):
        assert P.workspace_size(P.make_params(1, 2, 2, 1024, 64, sim_threshold=t)) == 0, t


def test_assign_rule_validated():
    p = P.make_params(1, 2, 2, 1024, 64, assign=P.ASSIGN_QUANTILE)
    assert P.workspace_size(p) > 0
    p.assign = 2
    assert P.workspace_size(p) == 0                                   # unknown rule


def test_forward_host_argument_errors_before_any_launch():
    p = P.make_params(1, 4, 2, 1024, 64)
    need = P.workspace_size(p)
    A, B = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)
    S1, S2, S3 = ctypes.c_void_p(0x1), ctypes.c_void_p(0x2), ctypes.c_void_p(0x3)
    f = lambda ws, groups, s1, s2, s3, hq=A: P.lib().psa_forward_host(
        ctypes.byref(p), hq, A, A, A, None, A, A, A, A, None, ws, need, groups, s1, s2, s3)
    assert f(B, 2, S1, S2, S2) == 1                                 # copy streams not distinct
    assert f(B, 2, S1, S1, S3) == 1
    assert f(B, 2, S1, S2, S3, hq=None) == 1                        # NULL host buffer
    assert f(B, 0, S1, S2, S3) == 1                                 # no groups
    assert f(B, 3, S1, S2, S3) == 1                                 # 3 groups cannot split 2 KV heads
    assert f(B, 8, S1, S2, S3) == 1                                 # more groups than query heads
    assert P.lib().psa_forward_host(ctypes.byref(p), A, A, A, A, None, A, A, A, A, None, B,
                                    need - 1, 2, S1, S2, S3) == 4   # workspace too small


def test_status_strings():
    for s in range(7):
        assert P.status_string(s)
    assert "timeout" in P.status_string(6)
