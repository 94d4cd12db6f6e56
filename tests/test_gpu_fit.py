"""Offline fit of the compression maps on the GPU (esa_gram, esa_fit_maps through the
C ABI) against the oracle (oracle/esa_fit.py), on the same bf16 calibration tokens.

The Gram matrix is compared entry by entry with the float64 product. The fitted maps
are unique only up to an invertible d' x d' transform (W_q T, W_k T^-T give the same
compressed scores), so the fit is compared on what is unique: the compressed scores
q~ . k~ of held-out tokens, which the least-squares optimum fixes whenever the d'-th
and (d'+1)-th singular values of C = Rq E Rk^T differ (they do here, though not by
much: the spectrum of the calibration recipe decays gradually, which is why the fit
oversamples its subspace and ends with a Rayleigh-Ritz step)."""
import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import esa as oesa
from oracle import esa_fit
from query_aware_selective_b200 import synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _scores(q, k, w_q, w_k):
    hq = q.shape[1]
    return oesa.compress(q, w_q, hq) @ oesa.compress(k, w_k, hq).T


@pytest.mark.parametrize("n,dim", [(1000, 384), (5000, 128), (128, 256), (70000, 1024)])
def test_gram_matches_float64(n, dim):
    g = torch.Generator().manual_seed(n + dim)
    x = torch.randn((n, dim), generator=g).to(torch.bfloat16)
    got = qas.gram(x.to(DEV)).cpu().numpy()
    qas.device_status()
    xd = x.double().numpy()
    ref = xd.T @ xd
    # bf16 products are exact in fp32; recursive fp32 summation of n terms errs by at
    # most (n - 1) 2^-24 times the sum of their magnitudes, which is at most the largest
    # diagonal entry here (|x_ri x_rj| <= (x_ri^2 + x_rj^2) / 2)
    tol = n * 2.0 ** -24 * np.abs(ref).max()
    assert np.abs(got - ref).max() <= tol
    assert np.array_equal(got, got.T)


def _fit_case(hq, hkv, d, n, rank, d_c, ridge, power_iters, seed, n_test=256, noise=0.1, oversample=32):
    oversample = min(oversample, hkv * d - d_c)
    w = synthetic.FitWorkload("case", hq, hkv, d, n, rank, d_c, oversample, noise, ridge, power_iters, seed)
    inp = synthetic.make_fit_inputs(w)
    w_q, w_k = qas.fit_maps(inp["q"].to(DEV), inp["k"].to(DEV), d_c, inp["omega"].to(DEV), ridge=ridge,
                            power_iters=power_iters)
    qas.device_status()
    q, k = inp["q"].double().numpy(), inp["k"].double().numpy()
    o_q, o_k = esa_fit.fit_maps(q, k, d_c, ridge=ridge)
    # held-out tokens of the same recipe (another seed)
    tq, tk = synthetic.make_calibration(hq, hkv, d, n_test, rank, seed + 100, noise)
    tq, tk = tq.double().numpy(), tk.double().numpy()
    got = _scores(tq, tk, w_q.double().cpu().numpy(), w_k.double().cpu().numpy())
    ref = _scores(tq, tk, o_q, o_k)
    return got, ref, (q, k, w_q, w_k, o_q, o_k)


@pytest.mark.parametrize("hq,hkv,d,n,rank,d_c,ridge", [
    (8, 2, 64, 4096, 16, 16, 0.0),        # GQA 4, 512 -> 16
    (4, 4, 64, 3000, 24, 24, 0.0),        # no GQA, ragged row count
    (8, 2, 64, 300, 16, 16, 1e-3),        # fewer tokens than dimensions: the ridge keeps it defined
])
def test_fit_scores_match_the_oracle(hq, hkv, d, n, rank, d_c, ridge):
    got, ref, _ = _fit_case(hq, hkv, d, n, rank, d_c, ridge, 8, seed=hq + n)
    assert np.abs(got - ref).max() <= 1e-4 * np.abs(ref).max()


def test_full_rank_fit_reproduces_the_merged_scores():
    # d' = Hkv * D: the compressed scores equal the merged-head scores exactly
    got, _, (q, k, *_rest) = _fit_case(4, 1, 128, 2048, 8, 128, 0.0, 2, seed=3, oversample=0)
    tq, tk = synthetic.make_calibration(4, 1, 128, 256, 8, 103, 0.1)
    full = esa_fit.scores_full(tq.double().numpy(), tk.double().numpy())
    assert np.abs(got - full).max() <= 1e-4 * np.abs(full).max()


def test_fit_loss_is_the_oracles():
    # the maps reach the oracle's least-squares loss on the calibration tokens
    _, _, (q, k, w_q, w_k, o_q, o_k) = _fit_case(8, 2, 64, 2048, 16, 16, 0.0, 8, seed=5)
    ours = esa_fit.fit_loss(q, k, w_q.double().cpu().numpy(), w_k.double().cpu().numpy())
    best = esa_fit.fit_loss(q, k, o_q, o_k)
    assert ours <= best * (1 + 1e-4)


def test_key_map_folds_back():
    # each group's rows of the expanded key map are equal: folding them (the packed
    # compression's sum over a group) gives the folded map B
    _, _, (q, k, w_q, w_k, *_r) = _fit_case(8, 2, 64, 2048, 16, 16, 0.0, 8, seed=6)
    wk = w_k.cpu().numpy().reshape(8, 64, 16)
    for g in range(2):
        for h in range(4 * g + 1, 4 * g + 4):
            assert np.array_equal(wk[h], wk[4 * g])


def test_not_positive_definite_is_reported():
    # fewer tokens than dimensions and no ridge: the Gram matrix is singular, a Cholesky
    # pivot is not positive, and the device status says so (no fault, the context stays)
    w = synthetic.FitWorkload("singular", 8, 2, 64, 100, 8, 8, 8, 0.1, 0.0, 1, 11)
    inp = synthetic.make_fit_inputs(w)
    qas.fit_maps(inp["q"].to(DEV), inp["k"].to(DEV), 8, inp["omega"].to(DEV))
    with pytest.raises(qas.EsaError, match="not positive"):
        qas.device_status()
    qas.device_status()                                  # read and cleared
    x = torch.ones((256, 128), dtype=torch.bfloat16, device=DEV)
    assert float(qas.gram(x)[0, 0]) == 256.0             # the context still works


def test_fit_full_workload_sampled():
    # the Llama-3-8B layer workload bench.py times: 65536 calibration tokens, 4096 -> 128
    w = synthetic.FIT_64K
    inp = synthetic.make_fit_inputs(w)
    w_q, w_k = qas.fit_maps(inp["q"].to(DEV), inp["k"].to(DEV), w.d_c, inp["omega"].to(DEV), ridge=w.ridge,
                            power_iters=w.power_iters)
    qas.device_status()
    q, k = inp["q"].double().numpy(), inp["k"].double().numpy()
    o_q, o_k = esa_fit.fit_maps(q, k, w.d_c, ridge=w.ridge)
    tq, tk = synthetic.make_calibration(w.hq, w.hkv, w.head_dim, 128, w.rank, w.seed + 100, w.noise)
    tq, tk = tq.double().numpy(), tk.double().numpy()
    got = _scores(tq, tk, w_q.double().cpu().numpy(), w_k.double().cpu().numpy())
    ref = _scores(tq, tk, o_q, o_k)
    assert np.abs(got - ref).max() <= 1e-4 * np.abs(ref).max()
    torch.cuda.empty_cache()
