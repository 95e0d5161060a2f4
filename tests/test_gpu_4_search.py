"""GPU vector search: tq_encode_vectors records are bit-exact against the
fp64 oracle (ties excepted), and tq_ip_search's top-k equals the oracle's
top-k over the GPU's own records, up to swaps of entries whose oracle scores
differ by at most 2e-3 * max|score|."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import (SEARCH_WORKLOADS, mixture_queries,
                                                            mixture_vectors)
from oracle import tq_oracle as O
from tests.tq_testutil import CodeReport, compare_codes, half_from_bits

pytestmark = pytest.mark.gpu
SWAP_TOL = 2e-3


def _padded(dim):
    d = 64
    while d < dim:
        d *= 2
    return d


def _oracle_codes(exp, dim, b_r, b_t, m):
    d = _padded(dim)
    cr, ct = O.unpack_codes(exp["codes"], d // 2, b_r, b_t)
    c = O.Codes(b_r=b_r, b_theta=b_t, s16=half_from_bits(exp["s16"]), cr=cr, ct=ct)
    c.rn16 = half_from_bits(exp["rn16"])
    c.bits = O.unpack_bits(exp["bits"], m)
    return c


def _check_topk(scores, idx, ref_scores, k):
    """GPU (scores, idx) [nq, k] against oracle scores [nq, n]: the returned
    entries are valid (each within tol of the oracle's k-th best, scores
    matching, no duplicates, descending) and complete (nothing scoring more
    than tol above the lowest returned entry was left out)."""
    swaps = 0
    for i in range(ref_scores.shape[0]):
        row = ref_scores[i]
        tol = SWAP_TOL * np.abs(row).max()
        order = np.lexsort((np.arange(row.size), -row))
        kth = row[order[k - 1]]
        got = idx[i]
        assert len(set(got.tolist())) == k, "duplicate indices"
        assert np.all(row[got] >= kth - tol), (i, row[got].min(), kth)
        # complete: every entry that beats the lowest returned one by more
        # than the tolerance was returned
        must = np.nonzero(row > row[got].min() + tol)[0]
        missing = set(must.tolist()) - set(got.tolist())
        assert not missing, (i, sorted(missing)[:5])
        np.testing.assert_allclose(scores[i], row[got], rtol=0, atol=tol)
        assert np.all(np.diff(scores[i]) <= tol)            # descending
        swaps += len(set(order[:k].tolist()) - set(got.tolist()))
    return swaps


def _build(n, dim, b_r=4, b_t=4, m=200, seed=0, nq=64, vec_seed=0):
    sw = SimpleNamespace(n=n, dim=dim, components=64)
    x = mixture_vectors(sw, vec_seed, 0, n)
    q = mixture_queries(SimpleNamespace(n=n, dim=dim, components=64, n_queries=nq), vec_seed, nq)
    idx = tq.TQVecIndex(dim, n, b_r, b_t, m, seed=seed, max_queries=max(nq, 1))
    idx.encode(torch.from_numpy(x).cuda())
    return idx, x, q


@pytest.mark.parametrize("dim,m", [(200, 200), (128, 128), (64, 64), (100, 24)])
def test_vector_encode_bit_exact(dim, m):
    n = 1500
    index, x, _ = _build(n, dim, m=m, nq=1)
    exp = index.export(0, n)
    d = _padded(dim)
    signs = O.rotation_signs(0, d)
    S = O.qjl_matrix(0, m, d)
    ref = O.encode(x.astype(np.float64), signs, S, 4, 4)
    shim = SimpleNamespace(head_dim=d, b_r=4, b_theta=4, qjl_bits=m)
    rep = CodeReport()
    rep.add(compare_codes({"k_codes": exp["codes"], "k_bits": exp["bits"], "k_s16": exp["s16"],
                           "k_rn16": exp["rn16"]}, ref, shim, True))
    print(rep)
    index.close()


@pytest.mark.parametrize("n,nq,k", [(6000, 70, 10), (100, 1, 1), (1000, 64, 16), (130, 3, 5)])
def test_search_topk_parity(n, nq, k):
    dim, m = 200, 200
    index, x, q = _build(n, dim, m=m, nq=nq)
    scores, idx = index.search(torch.from_numpy(q).cuda(), k=k)
    assert index.get_status() == 0
    scores, idx = scores.cpu().numpy(), idx.cpu().numpy()
    d = _padded(dim)
    codes = _oracle_codes(index.export(0, n), dim, 4, 4, m)
    ref = O.ip_scores(q.astype(np.float64), O.rotation_signs(0, d), O.qjl_matrix(0, m, d), codes)
    swaps = _check_topk(scores, idx, ref, k)
    print(f"n={n} nq={nq} k={k} tolerated swaps={swaps}")
    index.close()


@pytest.mark.parametrize("dim,m", [(64, 8), (100, 24), (128, 40), (128, 128), (256, 256)])
def test_search_qjl_step_shapes(dim, m):
    """Every QJL k-step arrangement: whole sign words, a last word with 8
    needed bits (one k-step), with 24 (two); two query tiles, the second
    ragged; a database that ends inside a round of 256."""
    n, nq, k = 1700, 130, 5
    index, x, q = _build(n, dim, m=m, nq=nq, vec_seed=2)
    scores, idx = index.search(torch.from_numpy(q).cuda(), k=k)
    assert index.get_status() == 0
    scores, idx = scores.cpu().numpy(), idx.cpu().numpy()
    d = _padded(dim)
    codes = _oracle_codes(index.export(0, n), dim, 4, 4, m)
    ref = O.ip_scores(q.astype(np.float64), O.rotation_signs(0, d), O.qjl_matrix(0, m, d), codes)
    _check_topk(scores, idx, ref, k)
    index.close()


def test_search_full_size_sampled_queries():
    """The full vector-search workload (1,000,000 x 200, 1024 queries, 4/4
    bits, m = 200, top-10) in the launch configuration the benchmark times;
    the oracle checks 4 sampled queries over all 10^6 records."""
    sw = SEARCH_WORKLOADS["vsearch"]
    index = tq.TQVecIndex(sw.dim, sw.n, sw.b_r, sw.b_theta, sw.qjl_bits, seed=0,
                          max_queries=sw.n_queries)
    chunk = 200_000
    for s in range(0, sw.n, chunk):
        index.encode(torch.from_numpy(mixture_vectors(sw, 0, s, min(chunk, sw.n - s))).cuda(), start=s)
    q = mixture_queries(sw, 0)
    scores, idx = index.search(torch.from_numpy(q).cuda(), k=sw.k)
    assert index.get_status() == 0
    scores, idx = scores.cpu().numpy(), idx.cpu().numpy()
    d = _padded(sw.dim)
    signs, S = O.rotation_signs(0, d), O.qjl_matrix(0, sw.qjl_bits, d)
    sample = [0, 1, 511, 1023]
    ref = np.empty((len(sample), sw.n))
    for s in range(0, sw.n, chunk):
        codes = _oracle_codes(index.export(s, min(chunk, sw.n - s)), sw.dim, sw.b_r, sw.b_theta,
                              sw.qjl_bits)
        ref[:, s:s + codes.s16.size] = O.ip_scores(q[sample].astype(np.float64), signs, S, codes)
    _check_topk(scores[sample], idx[sample], ref, sw.k)
    index.close()


def test_search_argument_checks():
    index, _, q = _build(200, 64, m=64, nq=4)
    qt = torch.from_numpy(q).cuda()
    with pytest.raises(tq.TQError):
        index.search(qt, k=17)          # k > 16
    with pytest.raises(tq.TQError):
        index.search(torch.cat([qt, qt]), k=3)    # more queries than max_queries
    index.close()
