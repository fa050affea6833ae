"""rb_gemv parity against the float64 oracle (dequantise, then multiply).

The GPU consumes the oracle's packed planes (uploaded), so a pack error cannot
hide a GEMV error; one end-to-end case also runs rb_pack -> rb_gemv.  Gates:
relative Frobenius error <= 2e-3 and a per-element bound (see cases.check_y).
Full-size workloads check every output where the oracle is fast enough and a
fixed sample of rows (first, last, ragged tail, random) otherwise.
"""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases

pytestmark = pytest.mark.gpu


def run_gemv(L, X, M, ydtype, flags=0, ws=None):
    N, K, k = L.n_out, L.k_in, L.k_planes
    if ws is None:
        ws = rbw.workspace(rbw.gemv_workspace_bytes(N, K, k, M))
    Xd = cases.to_dev(X)
    Y = rbw.gemv(L, Xd, ws=ws, flags=flags, y_dtype=ydtype)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy().astype(np.float64), ws


def per_elem(M, k):
    """Per-element gate factor: the byte-table path (M = 1, k <= 4) adds in fp32
    on the CUDA cores; the tensor-core path accumulates exact fp16 products in
    the MMA's fp32 accumulator, as rb_gemm does, and takes rb_gemm's factor."""
    return 1e-5 if (M == 1 and k <= 4) else 1e-4


def sample_rows(N, n=384, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(range(min(N, 64))) | set(range(max(0, N - 64), N))
    rows |= set(rng.choice(N, size=min(N, n), replace=False).tolist())
    return np.array(sorted(rows), np.int64)


CASES = [(0, 0, 1, 1), (1, 0, 2, 1), (1, 0, 2, 4), (1, 0, 2, 16), (2, 0, 2, 1), (2, 2, 2, 1),
         (2, 0, 2, 8), (3, 0, 1, 1), (3, 0, 2, 1), (3, 0, 2, 16), (3, 0, 1, 64)]


@pytest.mark.parametrize("wl,li,k,M", CASES)
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_gemv_workloads(wl, li, k, M, ydt):
    W, g, h = cases.layer_case(wl, li, k)
    N, K = W.shape
    planes, g16, h16 = cases.packed_case(wl, li, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations_for(synth.workload(wl), M, K)
    Yg, ws = run_gemv(L, X, M, ydt)
    rows = None if N * K * M <= 2 ** 27 else sample_rows(N)
    Yr = oracle.apply(planes, g16, h16, N, K, k, X, rows=rows)
    Yg = Yg if rows is None else Yg[:, rows]
    cases.check_y(Yg, Yr, cases.abs_bound(g16, h16, X, rows), bf16=ydt == torch.bfloat16, per_elem=per_elem(M, k))


@pytest.mark.parametrize("N,K,k,M", [(33, 288, 2, 1), (100, 800, 3, 1), (1, 32, 1, 1), (1000, 544, 4, 1),
                                     (70, 1056, 2, 2), (65, 320, 5, 3), (40, 256, 8, 17), (97, 2080, 2, 64),
                                     (31, 4096, 1, 5), (4097, 288, 2, 1), (97, 512, 6, 1), (300, 1024, 2, 9),
                                     (257, 4096, 2, 33), (1000, 2048, 4, 12), (8, 32, 1, 64)])
def test_gemv_ragged(N, K, k, M):
    rng = np.random.default_rng(N + 3 * K + 7 * k + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=8)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(M, K, seed=M + K)
    for ydt in (torch.float32, torch.bfloat16):
        Yg, _ = run_gemv(L, X, M, ydt)
        Yr = oracle.apply(planes, g16, h16, N, K, k, X)
        cases.check_y(Yg, Yr, cases.abs_bound(g16, h16, X), bf16=ydt == torch.bfloat16, per_elem=per_elem(M, k))


def test_gemv_deterministic_pdl_and_reused_workspace():
    W, g, h = cases.layer_case(1, 0, 2)
    N, K = W.shape
    planes, g16, h16 = cases.packed_case(1, 0, 2)
    L = cases.upload_layer(planes, g16, h16, N, K, 2)
    X = synth.activations(1, K, seed=123)
    ws = rbw.workspace(rbw.gemv_workspace_bytes(N, K, 2, 1))
    outs = [run_gemv(L, X, 1, torch.float32, flags=f, ws=ws)[0] for f in (0, rbw.RB_LAUNCH_PDL, 0, rbw.RB_LAUNCH_PDL)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_gemv_end_to_end_from_gpu_pack():
    """rb_pack -> rb_gemv on the device vs oracle.pack -> oracle.apply."""
    W, g, h = cases.layer_case(2, 2, 2)                 # down_proj 4096 x 11008
    N, K = W.shape
    L = rbw.pack(cases.to_dev(W), cases.to_dev(g), cases.to_dev(h), 2)
    X = synth.activations_for(synth.workload(2), 1, K)
    Yg, _ = run_gemv(L, X, 1, torch.float32)
    planes, g16, h16 = cases.packed_case(2, 2, 2)
    Yr = oracle.apply(planes, g16, h16, N, K, 2, X)
    cases.check_y(Yg, Yr, cases.abs_bound(g16, h16, X), bf16=False)


def test_gemv_errors_on_device():
    W, g, h = cases.layer_case(1, 0, 2)
    N, K = W.shape
    planes, g16, h16 = cases.packed_case(1, 0, 2)
    L = cases.upload_layer(planes, g16, h16, N, K, 2)
    X = cases.to_dev(synth.activations(65, K, seed=1))
    with pytest.raises(rbw.RbError) as e:
        rbw.gemv(L, X)                                  # M > 64
    assert e.value.status == rbw.RB_ERR_SHAPE
    Xbad = torch.zeros(2 * K + 8, dtype=torch.int16, device="cuda")[1:1 + K].view(1, K)   # 2-byte offset
    with pytest.raises(rbw.RbError) as e:
        rbw.gemv(L, Xbad)
    assert e.value.status == rbw.RB_ERR_ALIGN


@pytest.mark.parametrize("N,K,k,count", [(4096, 4096, 2, 5), (300, 800, 1, 3), (1000, 11008, 2, 2), (64, 256, 3, 130),
                                         (4096, 4096, 2, 48), (1024, 4096, 4, 33)])
def test_gemv_batch_matches_oracle_and_is_deterministic(N, K, k, count):
    """rb_gemv_batch over independent layers matches the oracle for every
    application (the launch shape, and so the association of the per-slice
    sums, depends on count), repeats bit for bit, and agrees with rb_gemv
    within the same bound."""
    rng = np.random.default_rng(N + K + count)
    layers, Xs, refs = [], [], []
    for j in range(min(count, 4)):
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        g, h = oracle.svid_greedy(W, k, iters=6)
        planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
        layers.append(cases.upload_layer(planes, g16, h16, N, K, k))
        Xs.append(synth.activations(1, K, seed=j + 7))
        refs.append((planes, g16, h16))
    idx = [j % len(layers) for j in range(count)]              # more applications than distinct layers
    Xd = [cases.to_dev(Xs[i]) for i in idx]
    Ys = [torch.empty(1, N, dtype=torch.float32, device="cuda") for _ in idx]
    Ys2 = [torch.empty(1, N, dtype=torch.float32, device="cuda") for _ in idx]
    rbw.gemv_batch([layers[i] for i in idx], Xd, Ys)
    rbw.gemv_batch([layers[i] for i in idx], Xd, Ys2)
    torch.cuda.synchronize()
    Yrefs = {}
    for j, i in enumerate(idx):
        assert torch.equal(Ys[j], Ys2[j]), "batch result not reproducible for application %d" % j
        if i not in Yrefs:
            planes, g16, h16 = refs[i]
            Yrefs[i] = (oracle.apply(planes, g16, h16, N, K, k, Xs[i]), cases.abs_bound(g16, h16, Xs[i]))
        Yr, bound = Yrefs[i]
        cases.check_y(Ys[j].cpu().numpy().astype(np.float64), Yr, bound, bf16=False)
        if j < len(layers):
            single = rbw.gemv(layers[i], Xd[j])
            torch.cuda.synchronize()
            cases.check_y(single.cpu().numpy().astype(np.float64), Yr, bound, bf16=False)


def test_gemv_batch_timed_launch_matches_oracle():
    """The benchmark's timed launch exactly: rb_gemv_batch over 96 distinct
    buffers of the 4096 x 4096 q_proj workload layer (k = 2, M = 1, fp32 out,
    programmatic dependent launch), one distinct activation row per
    application.  The batch plan picks the launch shape from the count, so this
    is the only way to check the association of per-slice sums that the bench
    times.  Every application is compared with the float64 oracle."""
    count, k = 96, 2
    W, g, h = cases.layer_case(1, 0, k)
    N, K = W.shape
    planes, g16, h16 = cases.packed_case(1, 0, k)
    base = cases.upload_layer(planes, g16, h16, N, K, k)
    layers = []
    for _ in range(count):
        L = rbw.PackedLayer(N, K, k)
        L.planes.copy_(base.planes)
        L.g16.copy_(base.g16)
        L.h16.copy_(base.h16)
        layers.append(L)
    X = synth.activations_for(synth.workload(1), count, K)          # one row per application
    Xd = cases.to_dev(X)
    Ys = [torch.empty(1, N, dtype=torch.float32, device="cuda") for _ in range(count)]
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    rbw.gemv_batch(layers, [Xd[j:j + 1] for j in range(count)], Ys, flags=rbw.RB_LAUNCH_PDL, dev_status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    Yr = oracle.apply(planes, g16, h16, N, K, k, X)
    bound = cases.abs_bound(g16, h16, X)
    for j in range(count):
        cases.check_y(Ys[j].cpu().numpy().astype(np.float64), Yr[j:j + 1], bound[j:j + 1], bf16=False)


@pytest.mark.parametrize("N,K,k,M,count", [(4096, 4096, 2, 4, 6), (4096, 4096, 2, 16, 3), (11008, 4096, 2, 8, 2),
                                           (300, 800, 3, 5, 7)])
def test_gemv_batch_multi_token(N, K, k, M, count):
    """rb_gemv_batch with M > 1 (one tensor-core launch for all layers) matches
    the oracle for every application and rb_gemv bit for bit (same launch
    shape per layer: the K split and token groups do not depend on count's
    effect on the grid beyond its size)."""
    rng = np.random.default_rng(N + K + M + count)
    layers, Xs, refs = [], [], []
    for j in range(min(count, 3)):
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        g, h = oracle.svid_greedy(W, k, iters=6)
        planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
        layers.append(cases.upload_layer(planes, g16, h16, N, K, k))
        Xs.append(synth.activations(M, K, seed=j + 11))
        refs.append((planes, g16, h16))
    idx = [j % len(layers) for j in range(count)]
    Xd = [cases.to_dev(Xs[i]) for i in idx]
    Ys = [torch.empty(M, N, dtype=torch.float32, device="cuda") for _ in idx]
    rbw.gemv_batch([layers[i] for i in idx], Xd, Ys)
    torch.cuda.synchronize()
    for j, i in enumerate(idx[:len(layers)]):
        planes, g16, h16 = refs[i]
        Yr = oracle.apply(planes, g16, h16, N, K, k, Xs[i])
        cases.check_y(Ys[j].cpu().numpy().astype(np.float64), Yr, cases.abs_bound(g16, h16, Xs[i]), bf16=False,
                      per_elem=per_elem(M, k))


@pytest.mark.parametrize("N,K,k,M", [(4096, 11008, 2, 64), (14336, 4096, 2, 48), (8192, 4096, 4, 40),
                                     (20000, 5152, 2, 40), (28672, 8192, 1, 32)])
def test_gemv_both_tensor_core_paths(N, K, k, M):
    """Above the measured crossover (N*K*k*M > 4.5e9, 32 <= M <= 64, k <= 4)
    rb_gemv runs the tcgen05 kernel when given its workspace (K split over a
    cluster; ragged N and K included) and the mma.sync kernel without one;
    both match the oracle on sampled rows."""
    rng = np.random.default_rng(N + K + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(M, K, seed=M + 5)
    rows = np.unique(np.concatenate([np.arange(40), np.arange(N - 40, N), rng.choice(N, 200, replace=False)]))
    Yr = oracle.apply(planes, g16, h16, N, K, k, X, rows=rows)
    bound = cases.abs_bound(g16, h16, X, rows=rows)
    assert rbw.gemv_workspace_bytes(N, K, k, M) > 0
    Xd = cases.to_dev(X)
    for ws in (rbw.workspace(rbw.gemv_workspace_bytes(N, K, k, M)), None):
        st = torch.zeros(4, dtype=torch.int32, device="cuda")
        Y = rbw.gemv(L, Xd, ws=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st[0].item()) == 0
        cases.check_y(Y.cpu().numpy().astype(np.float64)[:, rows], Yr, bound, bf16=False, per_elem=per_elem(M, k))


@pytest.mark.parametrize("N,K,k,M", [(4096, 4096, 2, 64), (300, 4096, 4, 33), (70, 1056, 2, 40), (4096, 4096, 1, 48)])
def test_gemv_small_layers_need_no_workspace(N, K, k, M):
    """Below the crossover the mma.sync kernel is the faster one: no workspace
    is asked for, and one passed anyway changes nothing."""
    assert rbw.gemv_workspace_bytes(N, K, k, M) == 0
    rng = np.random.default_rng(N + K + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    Xd = cases.to_dev(synth.activations(M, K, seed=M + 5))
    Ya = rbw.gemv(L, Xd)
    Yb = rbw.gemv(L, Xd, ws=rbw.workspace(1 << 20))
    torch.cuda.synchronize()
    assert torch.equal(Ya, Yb)


def test_gemv_batch_rejects_mixed_shapes():
    a = rbw.PackedLayer(64, 256, 2)
    b = rbw.PackedLayer(64, 512, 2)
    X = [torch.zeros(1, 256, dtype=torch.int16, device="cuda"), torch.zeros(1, 512, dtype=torch.int16, device="cuda")]
    Y = [torch.empty(1, 64, device="cuda") for _ in range(2)]
    with pytest.raises(rbw.RbError) as e:
        rbw.gemv_batch([a, b], X, Y)
    assert e.value.status == rbw.RB_ERR_SHAPE


def test_activation_overflow_is_reported_on_tensor_core_paths():
    """An activation that overflows the fp16 operand (|x| >= 65520) raises
    RB_DEV_RANGE on the mma.sync path (rb_gemv and rb_gemv_batch at M >= 2) and
    on the tcgen05 path; the byte-table path (M = 1) forms h*x in fp32 and
    raises nothing."""
    k = 2
    big = np.uint16(0x4789)                        # bf16 70144: finite, above fp16's range
    for M, ws, N, K in ((1, None, 256, 512), (4, None, 256, 512), (40, None, 256, 512), (48, "ws", 14336, 4096)):
        rng = np.random.default_rng(3)
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        g, h = oracle.svid_greedy(W, k, iters=2)
        planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
        L = cases.upload_layer(planes, g16, h16, N, K, k)
        X = synth.activations(M, K, seed=M)
        X[M - 1, 100] = big
        Xd = cases.to_dev(X)
        st = torch.zeros(4, dtype=torch.int32, device="cuda")
        w = rbw.workspace(rbw.gemv_workspace_bytes(N, K, k, M)) if ws else None
        rbw.gemv(L, Xd, ws=w, dev_status=st)
        torch.cuda.synchronize()
        assert int(st[0].item()) == (0 if M == 1 else rbw.RB_DEV_RANGE), (M, ws)
        if M > 1:
            st = torch.zeros(4, dtype=torch.int32, device="cuda")
            Ys = [torch.empty(M, N, device="cuda") for _ in range(2)]
            rbw.gemv_batch([L, L], [cases.to_dev(synth.activations(M, K, seed=9)), Xd], Ys, dev_status=st)
            torch.cuda.synchronize()
            assert int(st[0].item()) == rbw.RB_DEV_RANGE
