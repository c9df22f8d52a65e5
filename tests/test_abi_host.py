"""C-ABI checks that need no GPU: the library builds and loads, exports every
entry point declared in include/rlscan.h, and rejects bad arguments on the
host before any CUDA call (fake device addresses are never dereferenced)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rlscan.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RLSCAN_API\s+[\w\s\*]+?\b(rlscan_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib(rlscan_lib_path):
    # These tests hand the library fake device addresses that must be rejected
    # on the host; they are meant for a machine without a GPU, so that a
    # validation bug can never turn into a launch on real memory.
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("host-validation tests with fake pointers run only without a GPU")
    except ImportError:
        pass
    L = ctypes.CDLL(rlscan_lib_path)
    P, I64, F, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    L.rlscan_gae.argtypes = [P] * 7 + [I64, I64, F, F, P, SZ, P]
    L.rlscan_vtrace.argtypes = [P] * 9 + [I64, I64, F, F, F, F, P, SZ, P]
    L.rlscan_gae_with_returns.argtypes = [P] * 8 + [I64, I64, F, F, P, SZ, P]
    L.rlscan_gae_typed.argtypes = [P] * 8 + [I64, I64, F, F, ctypes.c_int, ctypes.c_int, P, SZ, P]
    L.rlscan_retrace.argtypes = [P] * 8 + [I64, I64, I64, F, F, F, P, SZ, P]
    L.rlscan_lambda_returns.argtypes = [P] * 7 + [I64, I64, F, F, P, SZ, P]
    L.rlscan_discounted_returns.argtypes = [P] * 6 + [I64, I64, F, P, SZ, P]
    L.rlscan_eligibility_traces.argtypes = [P] * 3 + [I64, I64, F, F, P, SZ, P]
    L.rlscan_episodic_prefix_sum.argtypes = [P, ctypes.c_int, P, P, I64, I64, P, SZ, P]
    L.rlscan_gae_noalloc.argtypes = [P] * 7 + [I64, I64, F, F, P]
    U = ctypes.c_uint
    L.rlscan_gae_ex.argtypes = [P] * 7 + [I64, I64, F, F, U, P, SZ, P]
    L.rlscan_retrace_ex.argtypes = [P] * 8 + [I64, I64, I64, F, F, F, U, P, SZ, P]
    L.rlscan_eligibility_traces_ex.argtypes = [P] * 3 + [I64, I64, F, F, U, P, SZ, P]
    L.rlscan_episodic_prefix_sum_ex.argtypes = [P, ctypes.c_int, P, P, I64, I64, U, P, SZ, P]
    L.rlscan_workspace_bytes.argtypes = [I64, I64]
    L.rlscan_workspace_bytes.restype = SZ
    L.rlscan_last_error.restype = ctypes.c_char_p
    L.rlscan_plan.argtypes = [I64, I64, I64, ctypes.POINTER(I64), ctypes.POINTER(ctypes.c_int),
                              ctypes.POINTER(ctypes.c_int), ctypes.POINTER(I64)]
    return L


def test_header_declares_the_seven_estimators():
    syms = declared_symbols()
    for est in ("gae", "vtrace", "retrace", "lambda_returns", "discounted_returns", "eligibility_traces",
                "episodic_prefix_sum"):
        assert f"rlscan_{est}" in syms


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(lib, s), f"{s} declared in rlscan.h but not exported"


def test_version(lib):
    # the library reports the version its header declares
    text = open(HEADER).read()
    declared = int(re.search(r"#define RLSCAN_VERSION (\d+)", text).group(1))
    assert lib.rlscan_version() == declared == 120


# fake, never-dereferenced device addresses, far apart
A, B, C, D, O1, O2 = (0x10000000 * k for k in range(1, 7))
E, T = 4, 128


def msg(lib):
    return lib.rlscan_last_error().decode()


def test_zero_sized_is_noop(lib):
    assert lib.rlscan_gae(None, None, None, None, None, None, None, 0, 128, 0.99, 0.95, None, 0, None) == OK
    assert lib.rlscan_gae(None, None, None, None, None, None, None, 8, 0, 0.99, 0.95, None, 0, None) == OK


@pytest.mark.parametrize("E_,T_", [(-1, 4), (4, -1)])
def test_negative_shape_rejected(lib, E_, T_):
    assert lib.rlscan_gae(A, B, C, None, None, None, O1, E_, T_, 0.99, 0.95, None, 0, None) == INVALID


def test_null_required_pointer_rejected(lib):
    assert lib.rlscan_gae(None, B, C, None, None, None, O1, E, T, 0.99, 0.95, None, 0, None) == INVALID
    assert "rewards" in msg(lib)
    assert lib.rlscan_gae(A, B, C, None, None, None, None, E, T, 0.99, 0.95, None, 0, None) == INVALID


def test_non_finite_parameters_rejected(lib):
    assert lib.rlscan_gae(A, B, C, None, None, None, O1, E, T, float("nan"), 0.95, None, 0, None) == INVALID
    assert lib.rlscan_vtrace(A, B, C, D, None, None, None, O1, O2, E, T, 0.99, 1.0, float("inf"), 1.0,
                             None, 0, None) == INVALID


def test_truncateds_need_bootstrap_values(lib):
    assert lib.rlscan_gae(A, B, C, D, None, None, O1, E, T, 0.99, 0.95, None, 0, None) == INVALID
    assert "bootstrap" in msg(lib)
    assert lib.rlscan_discounted_returns(A, C, D, None, None, O1, E, T, 0.99, None, 0, None) == INVALID


def test_output_overlapping_input_rejected(lib):
    # advantages starts inside values
    assert lib.rlscan_gae(A, B, C, None, None, None, B + 64, E, T, 0.99, 0.95, None, 0, None) == INVALID
    assert "overlaps" in msg(lib)
    # the two V-Trace outputs overlap each other
    assert lib.rlscan_vtrace(A, B, C, D, None, None, None, O1, O1 + 4, E, T, 0.99, 1.0, 1.0, 1.0,
                             None, 0, None) == INVALID


def test_retrace_argument_rules(lib):
    # truncateds is mandatory
    assert lib.rlscan_retrace(A, B, C, None, D, O2, None, O1, E, T, 1, 0.99, 0.95, 1.0, None, 0, None) == INVALID
    # probabilities required for A > 1
    assert lib.rlscan_retrace(A, B, C, None, D, O2, O2 + 0x1000000, O1, E, T, 18, 0.99, 0.95, 1.0,
                              None, 0, None) == INVALID
    assert lib.rlscan_retrace(A, B, C, None, D, O2, O2 + 0x1000000, O1, E, T, 0, 0.99, 0.95, 1.0,
                              None, 0, None) == INVALID
    assert lib.rlscan_retrace(A, B, C, C, D, O2, O2 + 0x1000000, O1, E, T, 97, 0.99, 0.95, 1.0,
                              None, 0, None) == UNSUPPORTED


def test_prefix_sum_dtype_rejected(lib):
    assert lib.rlscan_episodic_prefix_sum(A, 7, None, O1, E, T, None, 0, None) == UNSUPPORTED


def plan(lib, E_, T_, A_=1):
    te, th, lb, nt = ctypes.c_int64(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int64()
    assert lib.rlscan_plan(E_, T_, A_, ctypes.byref(te), ctypes.byref(th), ctypes.byref(lb), ctypes.byref(nt)) == OK
    return te.value, th.value, bool(lb.value), nt.value


@pytest.mark.parametrize("E_,T_", [(4096, 128), (64, 512), (4096, 32), (1024, 2048), (65536, 4096), (256, 1024)])
def test_plan_whole_rows_need_no_workspace(lib, E_, T_):
    tile, threads, lookback, ntiles = plan(lib, E_, T_)
    assert not lookback and tile % T_ == 0 and ntiles * tile >= E_ * T_
    assert tile == threads * (4 if tile == 512 else 8)


@pytest.mark.parametrize("E_,T_", [(16, 262144), (4096, 129), (3, 4097), (16, 4096)])
def test_plan_split_rows_need_workspace(lib, E_, T_):
    tile, threads, lookback, ntiles = plan(lib, E_, T_)
    assert lookback
    need = lib.rlscan_workspace_bytes(E_, T_)
    assert need >= 16 * ntiles


def test_missing_workspace_rejected(lib):
    # 16 x 262144 splits rows over tiles: a workspace is required
    assert lib.rlscan_gae(A, B, C, None, None, None, O1, 16, 262144, 0.99, 0.95, None, 0, None) == WORKSPACE
    _, _, lookback, ntiles = plan(lib, 16, 262144)
    need = 16 * ntiles  # what this call's plan needs: one 16-byte slot per tile
    assert lookback and lib.rlscan_workspace_bytes(16, 262144) >= need
    assert lib.rlscan_gae(A, B, C, None, None, None, O1, 16, 262144, 0.99, 0.95, D, need - 16, None) == WORKSPACE
    assert lib.rlscan_gae(A, B, C, None, None, None, O1, 16, 262144, 0.99, 0.95, D + 4, need, None) == WORKSPACE


def test_workspace_bytes_bounds(lib):
    assert lib.rlscan_workspace_bytes(0, 10) == 0
    assert lib.rlscan_workspace_bytes(-1, 10) == 0
    # whole rows: no call of this shape needs a workspace
    assert lib.rlscan_workspace_bytes(4096, 128) == 0
    assert lib.rlscan_workspace_bytes(16, 262144) > 0


def test_binding_imports_without_gpu():
    import linear_recurrence_scans_02_b200 as pkg
    assert callable(pkg.compute_gae) and callable(pkg.rlscan_gae)
    assert os.path.exists(pkg.library_path())


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    # 1 x (2^27 + 1) steps split over tiles needs about 2 MiB of scratch (one slot per 1024)
    T_big = (1 << 27) + 1
    far = [(k + 1) << 32 for k in range(4)]  # 512 MiB planes, 4 GiB apart: no overlap
    assert lib.rlscan_gae_noalloc(far[0], far[1], far[2], None, None, None, far[3], 1, T_big, 0.99, 0.95,
                                  None) == WORKSPACE
    assert "fixed scratch holds" in msg(lib)
    assert lib.rlscan_gae_noalloc(None, B, C, None, None, None, O1, 4, 128, 0.99, 0.95, None) == INVALID


def test_gae_with_returns_rejects_overlapping_outputs(lib):
    assert lib.rlscan_gae_with_returns(A, B, C, None, None, None, O1, O1 + 8, E, T, 0.99, 0.95, None, 0, None) == INVALID
    assert lib.rlscan_gae_with_returns(A, B, C, None, None, None, O1, None, E, T, 0.99, 0.95, None, 0, None) == INVALID
    assert lib.rlscan_gae_with_returns(A, B, C, None, None, None, O1, B, E, T, 0.99, 0.95, None, 0, None) == INVALID


def test_gae_typed_dtype_rules(lib):
    BF16, F16, U8, I32 = 2, 3, 4, 1
    assert lib.rlscan_gae_typed(A, B, C, None, None, None, O1, None, E, T, 0.99, 0.95, I32, U8, None, 0, None) == UNSUPPORTED
    assert lib.rlscan_gae_typed(A, B, C, None, None, None, O1, None, E, T, 0.99, 0.95, BF16, BF16, None, 0, None) == UNSUPPORTED
    # 2-byte values: planes of E*T*2 bytes; the output starting inside one is an overlap
    assert lib.rlscan_gae_typed(A, B, C, None, None, None, A + 2, None, E, T, 0.99, 0.95, BF16, U8, None, 0, None) == INVALID
    assert lib.rlscan_gae_typed(A, B, C, D, None, None, O1, None, E, T, 0.99, 0.95, F16, U8, None, 0, None) == INVALID


TIME_MAJOR, DONE_STARTS = 1, 2


def test_ex_option_bits(lib):
    # unknown bits, and the forward-only reset convention on a backward estimator
    for bad in (4, 0x80000000, DONE_STARTS, TIME_MAJOR | DONE_STARTS):
        assert lib.rlscan_gae_ex(A, B, C, None, None, None, O1, E, T, 0.99, 0.95, bad, None, 0, None) == INVALID
        assert "option" in msg(lib)
    assert lib.rlscan_eligibility_traces_ex(A, C, O1, E, T, 0.99, 0.95, 8, None, 0, None) == INVALID
    assert lib.rlscan_episodic_prefix_sum_ex(A, 0, C, O1, E, T, 16, None, 0, None) == INVALID
    # argument checks still run under the options
    assert lib.rlscan_gae_ex(None, B, C, None, None, None, O1, E, T, 0.99, 0.95, TIME_MAJOR, None, 0, None) == INVALID
    assert lib.rlscan_eligibility_traces_ex(A, C, A + 8, E, T, 0.99, 0.95, DONE_STARTS, None, 0, None) == INVALID


def test_ex_time_major_limits(lib):
    # multi-action Retrace has no time-major form
    assert lib.rlscan_retrace_ex(A, B, C, C, D, O2, O2 + 0x1000000, O1, E, T, 4, 0.99, 0.95, 1.0, TIME_MAJOR,
                                 None, 0, None) == UNSUPPORTED
    # E above the time-major limit ((8 + 1) E must stay below 2^31)
    E_big = (2 ** 31 - 1) // 9 + 1
    far = [(k + 1) << 33 for k in range(4)]  # ~1 GB planes, 8 GiB apart: no overlap
    assert lib.rlscan_gae_ex(far[0], far[1], far[2], None, None, None, far[3], E_big, 1, 0.99, 0.95, TIME_MAJOR,
                             None, 0, None) == UNSUPPORTED
    assert "time-major" in msg(lib)


class _Call(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("dtype", ctypes.c_int), ("flag_dtype", ctypes.c_int),
                ("options", ctypes.c_uint),
                ("E", ctypes.c_int64), ("T", ctypes.c_int64), ("A", ctypes.c_int64),
                ("gamma", ctypes.c_float), ("lambda_", ctypes.c_float), ("rho_bar", ctypes.c_float),
                ("c_bar", ctypes.c_float), ("inp", ctypes.c_void_p * 8), ("out", ctypes.c_void_p * 4),
                ("vtrace_lambda", ctypes.c_float)]


def _gae_call(r, v, d, out):
    c = _Call()
    c.kind, c.E, c.T, c.A, c.gamma, c.lambda_ = 1, E, T, 1, 0.99, 0.95
    c.inp[0], c.inp[1], c.inp[2], c.out[0] = r, v, d, out
    return c


def test_batch_host_rules(lib):
    lib.rlscan_batch.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert lib.rlscan_batch(None, 0, None, 0, None) == OK
    arr = (_Call * 2)()
    assert lib.rlscan_batch(arr, 17, None, 0, None) == INVALID
    assert lib.rlscan_batch(None, 1, None, 0, None) == INVALID
    arr[0] = _gae_call(A, B, C, O1)
    arr[0].kind = 99
    assert lib.rlscan_batch(arr, 1, None, 0, None) == INVALID
    assert "call 0" in msg(lib) and "kind" in msg(lib)
    # two calls writing one buffer: rejected before anything is launched
    arr[0] = _gae_call(A, B, C, O1)
    arr[1] = _gae_call(A, B, C, O1 + 64)
    assert lib.rlscan_batch(arr, 2, None, 0, None) == INVALID
    assert "calls 0 and 1" in msg(lib)
    # one call's output over the other call's input
    arr[1] = _gae_call(O1 + 8, B, C, O2)
    assert lib.rlscan_batch(arr, 2, None, 0, None) == INVALID
    # a call failing its own checks is named
    arr[1] = _gae_call(None, B, C, O2)
    assert lib.rlscan_batch(arr, 2, None, 0, None) == INVALID
    assert "call 1" in msg(lib) and "rewards" in msg(lib)


def test_batch_call_layout_matches_the_header(tmp_path):
    # compile a C probe of struct rlscan_call against include/rlscan.h and
    # compare its layout with the binding's ctypes mirror
    import subprocess
    import sys
    src = tmp_path / "lay.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "rlscan.h"\n'
                   'int main(void) { printf("%zu %zu %zu %zu %zu %zu %zu\\n", sizeof(rlscan_call), '
                   'offsetof(rlscan_call, E), offsetof(rlscan_call, gamma), offsetof(rlscan_call, c_bar), '
                   'offsetof(rlscan_call, in), offsetof(rlscan_call, out), offsetof(rlscan_call, vtrace_lambda)); '
                   'return 0; }\n')
    exe = tmp_path / "lay"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, "-o", str(exe), str(src)],
                   check=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    sys.path.insert(0, ROOT)
    from linear_recurrence_scans_02_b200.rlscan import _Call as Mirror
    want = [ctypes.sizeof(Mirror), Mirror.E.offset, Mirror.gamma.offset, Mirror.c_bar.offset, Mirror.inp.offset,
            Mirror.out.offset, Mirror.vtrace_lambda.offset]
    assert got == want
    assert [ctypes.sizeof(_Call), _Call.inp.offset] == [want[0], want[4]]


@pytest.mark.parametrize("E_,T_,tile,threads,lookback", [
    (4096, 128, 1024, 128, False),     # the 4096 x 128 workload: 128 threads x 8, whole rows
    (64, 512, 1024, 128, False),
    (4096, 2048, 2048, 256, False),    # a row needs a bigger tile to stay whole
    (256, 4096, 4096, 512, False),
    # rows that span tiles: the chunked two passes (128-thread blocks of
    # independent warps), reported as one workspace slot per 1024 elements
    (16, 262144, 1024, 128, True),     # long rows
    (1024, 8192, 1024, 128, True),
    (3, 70000, 1024, 128, True),
    (4096, 129, 1024, 128, True),       # rows not dividing any tile
])
def test_plan_choices(lib, E_, T_, tile, threads, lookback):
    # the launch plans the measurements in the design notes were taken with
    t, th, lb, nt = plan(lib, E_, T_)
    assert (t, th, lb) == (tile, threads, lookback)
    assert nt == -(-E_ * T_ // t)
