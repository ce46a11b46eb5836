"""The two-SM attention kernel (d = 128 on CTA pairs, cta_group::2) against the oracle.

The library runs it in place of the one-SM kernel while TSA_ATTEND_CTA_PAIRS is
set; these tests set it, re-run the d = 128 bf16 attention parity cases (all
rows on small shapes, ragged budgets, keep-all, scatter-add, block-sparse masks,
forced rescales, the 131072-token layer on sampled rows, dense K = L) and check
through the library's launch counter that the pair kernel is the one that ran.
"""

import pytest

import long_context_tsa_b200 as T

from . import test_gpu_fullsize as F
from . import test_gpu_parity as P

pytestmark = pytest.mark.gpu

D128 = [w for w in P.SMALL if w.D == 128 and w.dtype == "bf16"]


@pytest.fixture(autouse=True)
def cta_pairs(monkeypatch, request):
    monkeypatch.setenv("TSA_ATTEND_CTA_PAIRS", "1")
    before = T.tsa_debug_cta_pair_launch_count()
    yield
    if "d64_on_one_sm" not in request.node.name:
        assert T.tsa_debug_cta_pair_launch_count() > before, "the two-SM attention kernel did not run"


@pytest.mark.parametrize("w", D128, ids=lambda w: w.name)
def test_pairs_all_rows(w):
    P.test_attend_matches_oracle_all_rows(w)


@pytest.mark.parametrize("w", D128, ids=lambda w: w.name)
def test_pairs_ragged_budgets(w):
    P.test_attend_ragged_budgets_and_random_subsets(w)


@pytest.mark.parametrize("w", [w for w in P.SMALL[:3] if w in D128], ids=lambda w: w.name)
def test_pairs_keep_all_is_dense_causal(w):
    P.test_attend_keep_all_is_dense_causal(w)


@pytest.mark.parametrize("w", D128, ids=lambda w: w.name)
def test_pairs_forward(w):
    P.test_forward_matches_oracle(w)


@pytest.mark.parametrize("w", D128, ids=lambda w: w.name)
def test_pairs_accumulate(w):
    P.test_attend_accumulate_scatter_adds(w)


@pytest.mark.parametrize("w", D128, ids=lambda w: w.name)
@pytest.mark.parametrize("density", [0.0, 0.4, 1.0])
def test_pairs_block_sparse(w, density):
    P.test_attend_block_sparse_matches_oracle(w, density)


@pytest.mark.parametrize("spikes", [[0], [128 + 40], [384 + 70, 640 + 127]])
def test_pairs_logit_spikes(spikes):
    P.test_attend_logit_spikes_force_rescales(spikes)


def test_pairs_edge_shapes():
    P.test_edge_shapes()


def test_pairs_full_size_131072():
    # 205 chunks per group: an odd count, so the last pair's second CTA holds no rows.
    F.test_forward_full_size("gqa_bf16_L131072")


def test_pairs_dense_keep_all_131072():
    F.test_dense_keep_all_131072()


D64 = [w for w in P.SMALL if w.D == 64 and w.dtype == "bf16"]


@pytest.mark.parametrize("w", D64, ids=lambda w: w.name)
def test_pairs_request_leaves_d64_on_one_sm(w):
    # The two-SM kernel exists for d = 128 only: with the request set, d = 64
    # still runs (and matches the oracle) on the one-SM kernel.
    before = T.tsa_debug_cta_pair_launch_count()
    P.test_attend_matches_oracle_all_rows(w)
    assert T.tsa_debug_cta_pair_launch_count() == before
