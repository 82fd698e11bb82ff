"""The oracle against its pins (CPU only).  See tests/oracle_pins.py."""
import numpy as np
import pytest

import oracle
import workloads
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_oracle_rejects_table_entry_outside_pool():
    b = workloads.make_custom(30, [20], 2, 1, 16, 8, with_append=False)
    tables = b.block_tables.numpy().copy()
    tables[0, 1] = b.num_blocks
    with pytest.raises(oracle.OracleError, match="-2"):
        oracle.paged_decode(b.q, b.k_cache, b.v_cache, tables, b.context_lens.numpy(), 1, 8, b.scale)


def test_oracle_rejects_context_beyond_table():
    b = workloads.make_custom(31, [16], 2, 1, 16, 8, with_append=False)
    lens = np.array([17], dtype=np.int32)
    with pytest.raises(oracle.OracleError, match="-3"):
        oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), lens, 1, 8, b.scale)


def test_oracle_append_rejects_slot_outside_pool():
    b = workloads.make_custom(32, [4], 2, 1, 16, 8, with_append=False)
    with pytest.raises(oracle.OracleError, match="-2"):
        oracle.kv_append(b.k_cache, b.v_cache, b.k_new, b.v_new,
                         np.array([b.num_blocks * 8], dtype=np.int64), 8)


def test_oracle_sampled_rows_equal_full_rows():
    b = workloads.make_batch("tiny")
    full, _, _ = oracle.decode_step(b)
    pairs = [7, 0, 5]
    part, _, _ = oracle.decode_step(b, pairs=pairs)
    for k, flat in enumerate(pairs):
        assert np.array_equal(part[k], full[flat // 2, flat % 2])


def test_oracle_thread_count_does_not_change_result():
    b = workloads.make_batch("opt125m")
    a, _, _ = oracle.decode_step(b, pairs=list(range(0, 32 * 12, 17)), num_threads=1)
    c, _, _ = oracle.decode_step(b, pairs=list(range(0, 32 * 12, 17)), num_threads=4)
    assert np.array_equal(a, c)
