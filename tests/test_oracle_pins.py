"""The oracle against its pins (CPU only)."""
import pytest
import torch

from tests import pins


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda f: f.__name__)
def test_pin(oracle_lib, pin):
    pin(oracle_lib)


def test_thread_count_does_not_change_results(oracle_lib):
    q, k, v, k0, v0, seq = pins._rand_case(71, 2, 4, 4, 300)
    seq[1] = 123
    mask, _, _ = oracle_lib.route(q, k0, 0.6)
    o1, p1 = oracle_lib.decode(q, k, v, v0, seq, mask, n_threads=1)
    # fewer threads than units, between units and (unit, head) pairs, and more
    # than pairs: the oracle deals whole heads to its threads
    for nt in (4, 7, 13, 64):
        o4, p4 = oracle_lib.decode(q, k, v, v0, seq, mask, n_threads=nt)
        assert torch.equal(o1, o4) and torch.equal(torch.nan_to_num(p1), torch.nan_to_num(p4)), nt


def test_unit_subset_matches_full(oracle_lib):
    q, k, v, k0, v0, seq = pins._rand_case(72, 2, 4, 2, 90)
    mask, _, _ = oracle_lib.route(q, k0, 0.6)
    full, _ = oracle_lib.decode(q, k, v, v0, seq, mask)
    part, _ = oracle_lib.decode(q, k, v, v0, seq, mask, units=[1, 6])
    for u in (1, 6):
        b, g = divmod(u, 4)
        assert torch.equal(part[b, 2 * g:2 * g + 2], full[b, 2 * g:2 * g + 2])
    assert torch.isnan(part[0, 0]).all()


def test_rejects_bad_seq_len(oracle_lib):
    q, k, v, k0, v0, seq = pins._rand_case(73, 1, 2, 2, 8)
    mask = torch.zeros(2, dtype=torch.uint8)
    with pytest.raises(ValueError):
        oracle_lib.decode(q, k, v, v0, torch.tensor([0], dtype=torch.int32), mask)
    with pytest.raises(ValueError):
        oracle_lib.decode(q, k, v, v0, torch.tensor([9], dtype=torch.int32), mask)
