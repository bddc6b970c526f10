"""The C-ABI library loads, exports what include/km.h declares, and validates arguments before any CUDA work."""
import ctypes
import glob
import os
import re

import pytest

import flashassign_b200 as km

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"KM_API\s+[\w\s\*]+?\b(km_\w+)\s*\(", text))
    return names


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert {"km_assign", "km_sort_labels", "km_update", "km_lloyd", "km_status_string", "km_last_error",
            "km_device_fault"} <= names


def test_library_exports_every_declared_symbol():
    L = km.lib()
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared in include/ but not exported"
        assert name in km.SIGNATURES, f"{name} has no binding signature"


def test_status_strings():
    L = km.lib()
    for code in range(6):
        assert L.km_status_string(code)
    assert L.km_status_string(0) == b"ok"


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("args,expect", [
    (dict(X=None), 1),
    (dict(B=0), 1),
    (dict(N=-1), 1),
    (dict(K=0), 1),
    (dict(dtype=7), 1),
    (dict(d=12), 2),          # 24 bytes of fp16 per row: not a multiple of 16
    (dict(d=16392), 2),       # d > 16384
    (dict(B=70000), 2),
    (dict(K=1 << 24), 2),
    (dict(X=ctypes.c_void_p(0x10008)), 2),  # X not 16-byte aligned
])
def test_assign_rejects_bad_arguments_before_touching_the_device(args, expect):
    a = dict(X=FAKE, C=FAKE, B=2, N=100, K=10, d=64, dtype=km.KM_F16, labels=FAKE, mindist=None)
    a.update(args)
    rc = km.lib().km_assign(a["X"], a["C"], a["B"], a["N"], a["K"], a["d"], a["dtype"], a["labels"], a["mindist"],
                            None)
    assert rc == expect
    assert km.lib().km_last_error()


def test_update_rejects_misaligned_centroids_before_touching_the_device():
    rc = km.lib().km_update(FAKE, FAKE, 1, 64, 4, 16, km.KM_F32, FAKE, FAKE, ctypes.c_void_p(0x10004), None)
    assert rc == 2 and b"16-byte" in km.lib().km_last_error()


def test_update_and_sort_and_lloyd_reject_nulls():
    L = km.lib()
    assert L.km_update(None, FAKE, 1, 10, 2, 16, 0, FAKE, FAKE, FAKE, None) == 1
    assert L.km_sort_labels(FAKE, 1, 10, 2, None, FAKE, None, None) == 1
    assert L.km_lloyd(FAKE, FAKE, 1, 10, 2, 16, 0, -1, FAKE, FAKE, None, None) == 1
    assert L.km_device_fault(None, None) == 1
    assert L.km_lloyd_tol(FAKE, FAKE, 1, 10, 2, 16, 0, 5, 0.0, FAKE, FAKE, None, None, None) == 1
    assert L.km_lloyd_tol(FAKE, FAKE, 1, 10, 2, 16, 0, 5, -1.0, FAKE, FAKE, None, FAKE, None) == 1
    assert L.km_lloyd_tol(FAKE, FAKE, 1, 10, 2, 16, 0, 0, 0.0, FAKE, FAKE, None, FAKE, None) == 1
    assert L.km_assign_dense(None, FAKE, 1, 10, 2, 64, 1, FAKE, None, None) == 1
    assert L.km_update_scatter(FAKE, None, 1, 10, 2, 16, 0, FAKE, FAKE, FAKE, None) == 1
    assert L.km_assign_objective(FAKE, FAKE, 1, 10, 2, 16, 0, FAKE, None, None, None) == 1


def test_binding_raises_with_detail():
    with pytest.raises(km.KMError) as e:
        km.check("km_assign", km.lib().km_assign(None, FAKE, 1, 1, 1, 16, 0, FAKE, None, None))
    assert e.value.status == 1 and "non-null" in e.value.detail


def test_no_device_reports_a_cuda_error_instead_of_running():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a device is present: valid-looking fake pointers must not reach a kernel")
    rc = km.lib().km_assign(FAKE, FAKE, 1, 100, 10, 64, km.KM_F16, FAKE, None, None)
    assert rc == 4  # KM_E_CUDA from the device query
