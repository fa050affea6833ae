"""rb_gemm (tcgen05 tensor-core path) parity against the float64 oracle.

Prefill workloads run at their full sizes with sampled output rows and tokens
(first, last, ragged tails, random); ragged shapes cover N not a multiple of
128, M not a multiple of the token tile, K not a multiple of 64, every k the
kernel serves (1..4), and both output types.
"""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases

pytestmark = pytest.mark.gpu


def run_gemm(L, X, ydt, ws=None, dev_status=None):
    N, K, k = L.n_out, L.k_in, L.k_planes
    M = X.shape[0]
    ws = ws if ws is not None else rbw.workspace(rbw.gemm_workspace_bytes(N, K, k, M))
    Y = rbw.gemm(L, cases.to_dev(X), ws=ws, y_dtype=ydt, dev_status=dev_status)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy().astype(np.float64)


def sample(n, count, seed):
    rng = np.random.default_rng(seed)
    idx = set(range(min(n, 40))) | set(range(max(0, n - 40), n))
    idx |= set(rng.choice(n, size=min(n, count), replace=False).tolist())
    return np.array(sorted(idx), np.int64)


@pytest.mark.parametrize("wl,li,M", [(4, 0, 512), (4, 1, 512), (4, 0, 2048), (4, 1, 2048), (3, 0, 64)])
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_gemm_workloads(wl, li, M, ydt):
    w = synth.workload(wl)
    k = 2
    W, g, h = cases.layer_case(wl, li, k)
    N, K = W.shape
    planes, g16, h16 = cases.packed_case(wl, li, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations_for(w, M, K)
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    Yg = run_gemm(L, X, ydt, dev_status=st)
    assert int(st[0].item()) == 0
    rows, toks = sample(N, 300, 1), sample(M, 60, 2)
    Yr = oracle.apply(planes, g16, h16, N, K, k, X, rows=rows, toks=toks)
    bound = cases.abs_bound(g16, h16, X[toks], rows)
    cases.check_y(Yg[np.ix_(toks, rows)], Yr, bound, bf16=ydt == torch.bfloat16, per_elem=1e-4)


@pytest.mark.parametrize("N,K,k,M", [(128, 64, 1, 128), (200, 288, 2, 130), (33, 800, 3, 65), (300, 544, 4, 1),
                                     (4097, 256, 2, 7), (129, 1056, 1, 257), (64, 4096, 2, 300),
                                     (300, 512, 2, 1700), (257, 800, 1, 1100), (130, 544, 3, 1030)])
def test_gemm_ragged(N, K, k, M):
    rng = np.random.default_rng(N + K + 5 * k + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=8)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(M, K, seed=N + M)
    Yr = oracle.apply(planes, g16, h16, N, K, k, X)
    for ydt in (torch.float32, torch.bfloat16):
        Yg = run_gemm(L, X, ydt)
        cases.check_y(Yg, Yr, cases.abs_bound(g16, h16, X), bf16=ydt == torch.bfloat16, per_elem=1e-4)


@pytest.mark.parametrize("N,K,k,M", [(4097, 800, 2, 1000), (4000, 1056, 1, 2000), (2100, 544, 3, 1500),
                                     (1000, 4096, 4, 1300), (4096, 4096, 2, 2048), (300, 14336, 2, 9000)])
def test_gemm_many_tiles_match_oracle(N, K, k, M):
    """Grids of several waves (ragged rows, tokens and K; k = 1..4; a long K
    with a large M): sampled rows and tokens against the oracle."""
    rng = np.random.default_rng(N + K + 3 * k + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(M, K, seed=N + M + k)
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    for ydt in (torch.float32, torch.bfloat16):
        Yg = run_gemm(L, X, ydt, dev_status=st)
        assert int(st[0].item()) == 0
        rows, toks = sample(N, 200, 3), sample(M, 80, 4)
        Yr = oracle.apply(planes, g16, h16, N, K, k, X, rows=rows, toks=toks)
        cases.check_y(Yg[np.ix_(toks, rows)], Yr, cases.abs_bound(g16, h16, X[toks], rows),
                      bf16=ydt == torch.bfloat16, per_elem=1e-4)


def test_gemm_matches_gemv_small_m():
    """For M <= 64 both entry points compute the same product (to fp32 rounding)."""
    W, g, h = cases.layer_case(1, 0, 2)
    N, K = W.shape
    planes, g16, h16 = cases.packed_case(1, 0, 2)
    L = cases.upload_layer(planes, g16, h16, N, K, 2)
    X = synth.activations(16, K, seed=5)
    Yg = run_gemm(L, X, torch.float32)
    Yv = rbw.gemv(L, cases.to_dev(X), ws=rbw.workspace(rbw.gemv_workspace_bytes(N, K, 2, 16)))
    torch.cuda.synchronize()
    Yv = Yv.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(Yg - Yv) / np.linalg.norm(Yv) < 1e-5


@pytest.mark.parametrize("N,K,k,M", [(200, 544, 5, 77), (130, 1056, 6, 300), (64, 4096, 7, 33), (257, 800, 8, 129),
                                     (128, 13920, 8, 40), (300, 2080, 5, 1)])
def test_gemm_k5_to_8_matches_oracle(N, K, k, M):
    """k = 5..8 planes on the tensor cores (narrower token tiles, shorter
    pipeline; the k accumulators share tensor memory with the expansion
    stages), including the longest K whose h pairs fit shared memory at k = 8."""
    rng = np.random.default_rng(N + K + 7 * k + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=6)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(M, K, seed=N + M + k)
    Yr = oracle.apply(planes, g16, h16, N, K, k, X)
    for ydt in (torch.float32, torch.bfloat16):
        st = torch.zeros(4, dtype=torch.int32, device="cuda")
        Yg = run_gemm(L, X, ydt, dev_status=st)
        assert int(st[0].item()) == 0
        cases.check_y(Yg, Yr, cases.abs_bound(g16, h16, X), bf16=ydt == torch.bfloat16, per_elem=1e-4)


def test_gemm_k8_beyond_shared_memory_unsupported():
    N, K, k = 64, 14080, 8
    L = rbw.PackedLayer(N, K, k)
    with pytest.raises(rbw.RbError) as e:
        rbw.gemm(L, torch.zeros(8, K, dtype=torch.int16, device="cuda"),
                 ws=rbw.workspace(rbw.gemm_workspace_bytes(N, K, k, 8)))
    assert e.value.status == rbw.RB_ERR_UNSUPPORTED


@pytest.mark.parametrize("N,K,k,M", [(512, 1024, 2, 256), (300, 800, 3, 130)])
def test_gemm_wait_limit_expiry_reports_timeout_and_context_survives(N, K, k, M):
    """Bounded device waits (failure handling without a GPU fault): with a wait
    limit of 0 every pipeline stage that is not ready at its first probe ends
    the call; the kernel drains what it issued, frees its tensor memory and
    reports RB_DEV_TIMEOUT.  The next calls on the same stream (rb_gemm, and
    rb_gemm_wait_limit with a generous limit) then match the oracle."""
    rng = np.random.default_rng(N + K + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=6)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(M, K, seed=M)
    Xd = cases.to_dev(X)
    ws = rbw.workspace(rbw.gemm_workspace_bytes(N, K, k, M))
    Yr = oracle.apply(planes, g16, h16, N, K, k, X)
    bound = cases.abs_bound(g16, h16, X)
    for _ in range(2):
        st = torch.zeros(4, dtype=torch.int32, device="cuda")
        rbw.gemm_wait_limit(L, Xd, 0, ws=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st[0].item()) & rbw.RB_DEV_TIMEOUT
        st = torch.zeros(4, dtype=torch.int32, device="cuda")
        Y = rbw.gemm(L, Xd, ws=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st[0].item()) == 0
        cases.check_y(Y.cpu().numpy().astype(np.float64), Yr, bound, bf16=False, per_elem=1e-4)
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y = rbw.gemm_wait_limit(L, Xd, 500_000_000, ws=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    cases.check_y(Y.cpu().numpy().astype(np.float64), Yr, bound, bf16=False, per_elem=1e-4)
    with pytest.raises(rbw.RbError) as e:
        rbw.gemm_wait_limit(L, Xd, 2_000_000_000, ws=ws)
    assert e.value.status == rbw.RB_ERR_ARG


def test_gemm_wait_limit_expiry_many_ctas_then_correct():
    """The bounded-wait error path on a grid of several waves (4096 x 1024,
    M = 2048): limit 0 ends the call with RB_DEV_TIMEOUT after every CTA drains
    its loads and MMAs; the next rb_gemm on the stream matches the oracle on
    sampled outputs."""
    N, K, k, M = 4096, 1024, 2, 2048
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(M, K, seed=5)
    Xd = cases.to_dev(X)
    ws = rbw.workspace(rbw.gemm_workspace_bytes(N, K, k, M))
    rows, toks = sample(N, 200, 5), sample(M, 60, 6)
    Yr = oracle.apply(planes, g16, h16, N, K, k, X, rows=rows, toks=toks)
    bound = cases.abs_bound(g16, h16, X[toks], rows)
    for _ in range(2):
        st = torch.zeros(4, dtype=torch.int32, device="cuda")
        rbw.gemm_wait_limit(L, Xd, 0, ws=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st[0].item()) & rbw.RB_DEV_TIMEOUT
        st = torch.zeros(4, dtype=torch.int32, device="cuda")
        Y = rbw.gemm(L, Xd, ws=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st[0].item()) == 0
        Yg = Y.cpu().numpy().astype(np.float64)
        cases.check_y(Yg[np.ix_(toks, rows)], Yr, bound, bf16=False, per_elem=1e-4)
