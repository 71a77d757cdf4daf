"""The C-ABI library builds, loads and exports every entry point that
include/bcjr.h declares; host-side argument validation (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:BCJR_API\s+)?(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([A-Za-z_]\w*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("bcjr_soft_codeword", "bcjr_vjp", "viterbi_decode", "bcjr_posterior_argmax",
              "bcjr_get_device_error", "bcjr_launch_count", "bcjr_strerror", "bcjr_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from bcjr_sum_product_b200 import lib
    L = lib.load()
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(raw, name), name
    assert lib.version().count(".") == 2


def test_strerror_strings():
    from bcjr_sum_product_b200 import lib
    assert lib.strerror(0) == "ok"
    assert "invalid" in lib.strerror(1)
    assert "unsupported" in lib.strerror(2)
    assert "numerical" in lib.strerror(5)
    assert lib.strerror(99) == "unknown status"


def _call_soft(L=8, k=2, V=1, T=0.5, n_seq=1, length=8):
    from bcjr_sum_product_b200 import lib
    return lib.load().bcjr_soft_codeword(None, n_seq, length, L, k, V, None, float(T), None, None, None)


def test_shape_and_temperature_validation_without_gpu():
    from bcjr_sum_product_b200 import lib
    assert _call_soft(L=17) == lib.BCJR_ERR_UNSUPPORTED
    assert _call_soft(L=8, k=7, V=1) == lib.BCJR_ERR_UNSUPPORTED      # D > 6
    assert _call_soft(L=8, k=1, V=3, length=9) == lib.BCJR_ERR_UNSUPPORTED  # V not in {1,2,4}
    assert _call_soft(L=4, k=3, V=2) == lib.BCJR_ERR_INVALID_ARG      # D > L
    assert _call_soft(length=7, V=2) == lib.BCJR_ERR_INVALID_ARG      # len % V
    assert _call_soft(length=0) == lib.BCJR_ERR_INVALID_ARG
    assert _call_soft(length=8193) == lib.BCJR_ERR_UNSUPPORTED
    assert _call_soft(T=0.0) == lib.BCJR_ERR_INVALID_ARG
    assert _call_soft(T=float("nan")) == lib.BCJR_ERR_INVALID_ARG
    assert _call_soft(T=float("inf")) == lib.BCJR_ERR_INVALID_ARG
    assert _call_soft(T=-1.0) == lib.BCJR_ERR_INVALID_ARG
    assert _call_soft(n_seq=-1) == lib.BCJR_ERR_INVALID_ARG
    # valid shape but null codebook
    assert _call_soft() == lib.BCJR_ERR_INVALID_ARG
    L = lib.load()
    assert L.viterbi_decode(None, 1, 8, 17, 2, 1, None, None, None, None) == lib.BCJR_ERR_UNSUPPORTED
    assert L.bcjr_vjp(None, 1, 8, 8, 2, 1, None, 0.5, None, None, None, None, None) == lib.BCJR_ERR_INVALID_ARG
    assert L.bcjr_posterior_argmax(None, 1, 8, 8, 2, 1, None, -2.0, None, None) == lib.BCJR_ERR_INVALID_ARG
    qat = L.bcjr_qat_step
    assert qat(None, None, 1, 8, 17, 2, 1, None, 0.5, 1e-3, 0.0, None, None, None, None, None) == lib.BCJR_ERR_UNSUPPORTED
    assert qat(None, None, 1, 8, 8, 2, 1, None, 0.0, 1e-3, 0.0, None, None, None, None, None) == lib.BCJR_ERR_INVALID_ARG
    assert qat(None, None, 1, 8, 8, 2, 1, None, 0.5, float("nan"), 0.0, None, None, None, None, None) == lib.BCJR_ERR_INVALID_ARG
    assert qat(None, None, 1, 8, 8, 2, 1, None, 0.5, 1e-3, float("inf"), None, None, None, None, None) == lib.BCJR_ERR_INVALID_ARG
    assert qat(None, None, 1, 8, 8, 2, 1, None, 0.5, 1e-3, 0.0, None, None, None, None, None) == lib.BCJR_ERR_INVALID_ARG


def test_binding_rejects_host_tensors():
    import torch
    from bcjr_sum_product_b200 import lib
    with pytest.raises(TypeError):
        lib.soft_codeword(torch.zeros(2, 8), torch.zeros(256), 8, 2, 1, 0.5)


def test_rejected_calls_launch_nothing():
    """bcjr_launch_count counts kernels issued: calls that fail argument or
    shape validation (no GPU needed) leave it unchanged."""
    from bcjr_sum_product_b200 import lib
    n0 = lib.launch_count()
    assert n0 >= 0
    assert _call_soft(L=17) == lib.BCJR_ERR_UNSUPPORTED
    assert _call_soft(length=0) == lib.BCJR_ERR_INVALID_ARG
    assert lib.launch_count() == n0
