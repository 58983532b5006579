"""The CPU oracle pinned to facts that do not come from the oracle itself (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import pins


def oracle_impl(q, k, v, g, beta, h0):
    return oracle.recurrent(q, k, v, g, beta, h0)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle_impl)


def test_oracle_threads_do_not_change_results():
    rng = np.random.default_rng(11)
    case = pins.rand_case(rng, B=3, T=33, Hk=2, Hv=4, Dk=8, Dv=8, gate="channel")
    o1, s1 = oracle.recurrent(*case, nthreads=1)
    o4, s4 = oracle.recurrent(*case, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(s1, s4)


def test_oracle_no_h0_means_zero_state():
    rng = np.random.default_rng(12)
    q, k, v, g, beta, h0 = pins.rand_case(rng, T=9, Dk=4, Dv=4)
    o1, s1 = oracle.recurrent(q, k, v, g, beta, None)
    o2, s2 = oracle.recurrent(q, k, v, g, beta, np.zeros_like(h0))
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_oracle_rejects_bad_heads():
    rng = np.random.default_rng(13)
    q, k, v, g, beta, h0 = pins.rand_case(rng, Hk=2, Hv=3)
    with pytest.raises(ValueError):
        oracle.recurrent(q, k, v, g, beta, h0)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T", [16, 100, 256])
def test_chunked_matches_recurrent(paper_facts, gate, T):
    """Exact chunkwise form vs the 64-bit token recurrence at the chunk sizes and the bound
    the SinkProbe README states, outputs and memory (state) both, with a ragged tail
    whenever T is not a multiple of the chunk size."""
    spec = paper_facts["chunkwise_check"]
    rng = np.random.default_rng(T + (gate == "channel"))
    case = pins.rand_case(rng, B=1, T=T, Hk=1, Hv=3, Dk=16, Dv=8, gate=gate)
    o_ref, s_ref = oracle.recurrent(*case)
    for C in spec["chunk_sizes"]:
        o, s = oracle.chunked(*case, chunk=C)
        assert np.max(np.abs(o - o_ref)) <= spec["max_abs_diff"], C
        assert np.max(np.abs(s - s_ref)) <= spec["max_abs_diff"], C


def test_grouped_heads_at_the_pages_ratio(paper_facts):
    """16 key heads shared by 48 value heads: each key head serves 3 value heads."""
    gh = paper_facts["grouped_value_heads"]
    rep = gh["value_heads"] // gh["key_heads"]
    pins.pin_grouped_heads(oracle_impl, seed=21, Hk=2, Hv=2 * rep)


def test_decode_steps_equal_one_long_sequence():
    """Repeated single-token steps with state carried equal the T-token recurrence."""
    rng = np.random.default_rng(14)
    q, k, v, g, beta, h0 = pins.rand_case(rng, B=2, T=7, Hk=1, Hv=2, Dk=4, Dv=3)
    o_ref, s_ref = oracle.recurrent(q, k, v, g, beta, h0)
    sw = lambda x: np.ascontiguousarray(np.swapaxes(x, 0, 1))
    o, s = oracle.decode_steps(sw(q), sw(k), sw(v), sw(g), sw(beta), h0)
    assert np.array_equal(sw(o), o_ref) and np.array_equal(s, s_ref)
