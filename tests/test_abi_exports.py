"""Host-side checks of the C ABI (no GPU needed).

* librbw.so loads and exports every function declared in include/rbw.h, and
  the Python binding describes exactly that set.
* Size helpers agree with the oracle's independent size formula.
* Argument errors are returned before any CUDA call, and a valid call on a
  machine without a B200 fails loudly (RB_ERR_UNSUPPORTED), never silently.
"""
import ctypes
import os
import re
import types

import pytest
import torch

import oracle
from residual_binarized_weight_b200 import build as rbw_build
from residual_binarized_weight_b200 import rbw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rbw.h")


@pytest.fixture(scope="module")
def L():
    rbw_build.build()
    return rbw.lib()


def declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return set(re.findall(r"\b(rb_[a-z0-9_]+)\s*\(", txt))


def test_exports_match_header(L):
    decl = declared_functions()
    assert decl, "no declarations parsed"
    assert decl == set(rbw.SIGNATURES), decl ^ set(rbw.SIGNATURES)
    for name in decl:
        assert hasattr(L, name), name


def test_version_and_status_strings(L):
    assert L.rb_version() >= 100
    for code in range(7):
        assert L.rb_status_string(code).decode().startswith("RB_")


@pytest.mark.parametrize("N,K,k", [(256, 512, 1), (4096, 4096, 2), (33, 288, 3), (1, 32, 8), (11008, 4096, 2)])
def test_packed_words_matches_oracle(L, N, K, k):
    assert L.rb_packed_words(N, K, k) == oracle.plane_words(N, K, k)


def test_size_helpers_reject_bad_shapes(L):
    assert L.rb_packed_words(4, 48, 1) == 0
    assert L.rb_packed_words(0, 64, 1) == 0
    assert L.rb_packed_words(4, 64, 9) == 0
    assert L.rb_gemv_workspace_bytes(4096, 4096, 2, 1) == 0   # partial sums stay on chip
    assert L.rb_gemm_workspace_bytes(4096, 4096, 2, 64) >= 64 * 4096 * 2
    assert L.rb_gemm_workspace_bytes(4096, 4096, 8, 64) > 0   # the tensor-core path serves k <= 8
    assert L.rb_gemm_workspace_bytes(4096, 4096, 9, 64) == 0
    assert L.rb_qat_backward_workspace_bytes(100, 512, 2) == 0  # N must be a multiple of 32
    assert L.rb_qat_backward_workspace_bytes(4096, 4096, 2) > 0
    assert L.rb_rowmajor_words(4096, 4096, 2) == 2 * 4096 * 128
    assert L.rb_svid_workspace_bytes(4096, 4096) > 0
    # rb_gemv takes the tcgen05 path (and asks for a workspace) only above the crossover
    assert L.rb_gemv_workspace_bytes(4096, 4096, 2, 64) == 0
    assert L.rb_gemv_workspace_bytes(14336, 4096, 2, 64) > 0
    assert L.rb_gemv_workspace_bytes(14336, 4096, 2, 16) == 0
    assert L.rb_gemv_workspace_bytes(14336, 4096, 5, 64) == 0
    # training forward: the planes (256-byte aligned) in front of rb_gemm's workspace
    pb = (L.rb_packed_words(4096, 4096, 2) * 4 + 255) // 256 * 256
    assert L.rb_qat_forward_workspace_bytes(4096, 4096, 2, 2048) == pb + L.rb_gemm_workspace_bytes(4096, 4096, 2, 2048)
    assert L.rb_qat_forward_workspace_bytes(4096, 4096, 9, 2048) == 0


def test_codebook_size_helpers_match_the_oracle(L):
    for c in (1, 2, 3, 255, 256, 257, 7132, 65535, 65536):
        assert L.rb_btc_index_bits(c) == oracle.btc_index_bits(c)
    assert L.rb_btc_index_bits(0) == 0 and L.rb_btc_index_bits(65537) == 0
    for K, w in ((4096, 13), (544, 7), (32, 1), (8192, 16)):
        assert L.rb_btc_row_words(K, w) == oracle.btc_row_words(K, w)
    assert L.rb_btc_row_words(48, 13) == 0
    assert L.rb_btc_gemv_workspace_bytes(4096, 4096) == 16 * 4096 * 4            # one partial per slice and row
    assert L.rb_btc_gemv_batch_workspace_bytes(4096, 4096, 100) == 64 * 16 * 4096 * 4  # groups of 64 layers
    assert L.rb_btc_encode_workspace_bytes(7132) > 65536 * 16
    assert L.rb_btc_encode_workspace_bytes(0) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


# A call that passes every argument check launches kernels on a machine with a
# GPU, so the calls below that do (made-up device addresses, expecting
# RB_ERR_UNSUPPORTED) run only where no CUDA device is visible.  The
# argument-error calls return before any CUDA call and run everywhere.
no_device = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="well-formed calls with made-up pointers would launch kernels")


def test_pack_argument_errors_on_host(L):
    a = _fake(0x10000)
    assert L.rb_pack(None, a, a, 4, 64, 1, a, a, a, None, None) == rbw.RB_ERR_ARG
    assert L.rb_pack(a, a, a, 4, 64, 0, a, a, a, None, None) == rbw.RB_ERR_ARG
    assert L.rb_pack(a, a, a, 4, 48, 1, a, a, a, None, None) == rbw.RB_ERR_SHAPE
    assert L.rb_pack(a, a, a, 0, 64, 1, a, a, a, None, None) == rbw.RB_ERR_SHAPE
    assert L.rb_pack(_fake(0x10004), a, a, 4, 64, 1, a, a, a, None, None) == rbw.RB_ERR_ALIGN


def test_apply_argument_errors_on_host(L):
    a = _fake(0x10000)
    lay = rbw.RbLayer(64, 256, 2, 0, 0x10000, 0x10000, 0x10000)
    for fn in (L.rb_gemv, L.rb_gemm):
        assert fn(None, a, 1, a, 0, None, 0, None, 0, None) == rbw.RB_ERR_ARG
        assert fn(ctypes.byref(lay), a, 1, a, 7, None, 0, None, 0, None) == rbw.RB_ERR_ARG
        assert fn(ctypes.byref(lay), a, 0, a, 0, None, 0, None, 0, None) == rbw.RB_ERR_SHAPE
        assert fn(ctypes.byref(lay), _fake(0x10002), 1, a, 0, None, 0, None, 0, None) == rbw.RB_ERR_ALIGN
        bad = rbw.RbLayer(64, 250, 2, 0, 0x10000, 0x10000, 0x10000)
        assert fn(ctypes.byref(bad), a, 1, a, 0, None, 0, None, 0, None) == rbw.RB_ERR_SHAPE
        res = rbw.RbLayer(64, 256, 2, 1, 0x10000, 0x10000, 0x10000)
        assert fn(ctypes.byref(res), a, 1, a, 0, None, 0, None, 0, None) == rbw.RB_ERR_ARG
    assert L.rb_gemm(ctypes.byref(lay), a, 1, a, 0, None, 0, None, 0, None) == rbw.RB_ERR_WORKSPACE
    assert L.rb_gemv(ctypes.byref(lay), a, 65, a, 0, None, 0, None, 0, None) == rbw.RB_ERR_SHAPE
    assert L.rb_gemv(ctypes.byref(lay), a, 1, a, 0, None, 0, None, 2, None) == rbw.RB_ERR_ARG


def test_transpose_argument_errors_on_host(L):
    lay = rbw.RbLayer(64, 256, 2, 0, 0x10000, 0x10000, 0x10000)
    dst = _fake(0x100000)
    assert L.rb_transpose_planes(None, dst, None) == rbw.RB_ERR_ARG
    assert L.rb_transpose_planes(ctypes.byref(lay), None, None) == rbw.RB_ERR_ARG
    ragged_n = rbw.RbLayer(48, 256, 2, 0, 0x10000, 0x10000, 0x10000)    # N becomes the input width
    assert L.rb_transpose_planes(ctypes.byref(ragged_n), dst, None) == rbw.RB_ERR_SHAPE
    assert L.rb_transpose_planes(ctypes.byref(lay), _fake(0x100008), None) == rbw.RB_ERR_ALIGN
    # 2 planes x 1 slice x 2 tiles = 4 KB from 0x10000: a destination inside it overlaps
    assert L.rb_transpose_planes(ctypes.byref(lay), _fake(0x10400), None) == rbw.RB_ERR_ARG


def test_svid_argument_errors_on_host(L):
    a = _fake(0x10000)
    assert L.rb_svid_greedy(a, 4, 64, 1, 20, a, a, None, 0, None) == rbw.RB_ERR_ARG
    assert L.rb_svid_greedy(a, 4, 64, 1, 0, a, a, a, 1 << 20, None) == rbw.RB_ERR_ARG
    assert L.rb_svid_greedy(a, 4, 40, 1, 20, a, a, a, 1 << 20, None) == rbw.RB_ERR_SHAPE
    assert L.rb_svid_greedy(a, 4, 64, 1, 20, a, a, a, 16, None) == rbw.RB_ERR_WORKSPACE


def test_training_forward_argument_errors_on_host(L):
    a = _fake(0x10000)
    ws = L.rb_qat_forward_workspace_bytes(64, 256, 2, 8)
    assert L.rb_qat_forward(None, a, a, 64, 256, 2, a, 8, a, 0, a, ws, None, 0, None) == rbw.RB_ERR_ARG
    assert L.rb_qat_forward(a, a, a, 64, 256, 9, a, 8, a, 0, a, ws, None, 0, None) == rbw.RB_ERR_ARG
    assert L.rb_qat_forward(a, a, a, 64, 248, 2, a, 8, a, 0, a, ws, None, 0, None) == rbw.RB_ERR_SHAPE
    assert L.rb_qat_forward(_fake(0x10004), a, a, 64, 256, 2, a, 8, a, 0, a, ws, None, 0, None) == rbw.RB_ERR_ALIGN
    assert L.rb_qat_forward(a, a, a, 64, 256, 2, a, 8, a, 0, a, ws - 16, None, 0, None) == rbw.RB_ERR_WORKSPACE


def test_codebook_argument_errors_on_host(L):
    a = _fake(0x10000)
    lay = rbw.RbLayer(64, 256, 2, 0, 0x10000, 0x10000, 0x10000)
    ws = L.rb_btc_encode_workspace_bytes(16)
    enc = L.rb_btc_encode
    assert enc(None, 0, 16, 2, a, None, a, a, ws, None) == rbw.RB_ERR_ARG
    assert enc(ctypes.byref(lay), 2, 16, 2, a, None, a, a, ws, None) == rbw.RB_ERR_ARG        # plane >= k
    assert enc(ctypes.byref(lay), 0, 0, 2, a, None, a, a, ws, None) == rbw.RB_ERR_ARG         # c_max
    bad = rbw.RbLayer(64, 248, 2, 0, 0x10000, 0x10000, 0x10000)
    assert enc(ctypes.byref(bad), 0, 16, 2, a, None, a, a, ws, None) == rbw.RB_ERR_SHAPE
    assert enc(ctypes.byref(lay), 0, 16, 2, _fake(0x10001), None, a, a, ws, None) == rbw.RB_ERR_ALIGN
    assert enc(ctypes.byref(lay), 0, 16, 2, a, None, a, a, ws - 16, None) == rbw.RB_ERR_WORKSPACE
    blay = rbw.RbBtcLayer(64, 256, 2, 16, 4, 0, 0x10000, 0x10000, 0x10000, 0x10000)
    wsg = L.rb_btc_gemv_workspace_bytes(64, 256)
    assert L.rb_btc_gemv(None, a, a, 0, a, wsg, None, 0, None) == rbw.RB_ERR_ARG
    wrong_w = rbw.RbBtcLayer(64, 256, 2, 16, 5, 0, 0x10000, 0x10000, 0x10000, 0x10000)
    assert L.rb_btc_gemv(ctypes.byref(wrong_w), a, a, 0, a, wsg, None, 0, None) == rbw.RB_ERR_ARG
    k3 = rbw.RbBtcLayer(64, 256, 3, 16, 4, 0, 0x10000, 0x10000, 0x10000, 0x10000)
    assert L.rb_btc_gemv(ctypes.byref(k3), a, a, 0, a, wsg, None, 0, None) == rbw.RB_ERR_UNSUPPORTED
    assert L.rb_btc_gemv(ctypes.byref(blay), a, a, 0, a, wsg - 16, None, 0, None) == rbw.RB_ERR_WORKSPACE


@no_device
def test_well_formed_calls_fail_loudly_without_a_device(L):
    """Calls that pass every argument check return RB_ERR_UNSUPPORTED when no
    sm_100 device is current: nothing runs on the CPU instead."""
    a = _fake(0x10000)
    lay = rbw.RbLayer(64, 256, 2, 0, 0x10000, 0x10000, 0x10000)
    assert L.rb_pack(a, a, a, 4, 64, 1, a, a, a, None, None) == rbw.RB_ERR_UNSUPPORTED
    for fn in (L.rb_gemv, L.rb_gemm):
        assert fn(ctypes.byref(lay), a, 1, a, 0, a, 1 << 30, None, 0, None) == rbw.RB_ERR_UNSUPPORTED
    assert L.rb_transpose_planes(ctypes.byref(lay), _fake(0x100000), None) == rbw.RB_ERR_UNSUPPORTED
    assert L.rb_svid_greedy(a, 4, 64, 1, 20, a, a, a, 1 << 20, None) == rbw.RB_ERR_UNSUPPORTED
    assert L.rb_qat_forward(a, a, a, 64, 256, 2, a, 8, a, 0, a, 1 << 30, None, 0, None) == rbw.RB_ERR_UNSUPPORTED
    assert L.rb_btc_encode(ctypes.byref(lay), 0, 16, 2, a, None, a, a, 1 << 30, None) == rbw.RB_ERR_UNSUPPORTED
    blay = rbw.RbBtcLayer(64, 256, 2, 16, 4, 0, 0x10000, 0x10000, 0x10000, 0x10000)
    assert L.rb_btc_gemv(ctypes.byref(blay), a, a, 0, a, 1 << 30, None, 0, None) == rbw.RB_ERR_UNSUPPORTED


def test_product_does_not_import_oracle():
    """The CUDA binding, build script and package never reference the oracle."""
    pkg = os.path.join(ROOT, "residual_binarized_weight_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "rb_oracle" not in txt, f


@no_device
def test_binding_fails_loudly_without_a_device():
    """The binding marshals host tensors' pointers and the library refuses to
    run without an sm_100 device: no CPU fallback."""
    L = rbw.PackedLayer(64, 256, 2, "cpu")
    with pytest.raises(rbw.RbError) as e:
        rbw.transpose(L, stream=types.SimpleNamespace(cuda_stream=0))
    assert e.value.status == rbw.RB_ERR_UNSUPPORTED
    X = torch.zeros(1, 256, dtype=torch.int16)
    with pytest.raises(rbw.RbError) as e:
        rbw.gemv(L, X, Y=torch.empty(1, 64), stream=types.SimpleNamespace(cuda_stream=0))
    assert e.value.status == rbw.RB_ERR_UNSUPPORTED
