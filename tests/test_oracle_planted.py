"""Plant plausible mistakes in the oracle (on the CPU, by monkeypatching) and
check that the pins in ``test_oracle_pins`` catch every one of them.

This shows the pins constrain the oracle: a dropped scale, a missing max
subtraction, a wrong GQA mapping, a wrong in-block offset, a transposed
operand or a merge without the max rescale each fails at least one pin.
"""

import numpy as np
import pytest

import oracle.attention as oa
import oracle.paging as op
from tests import test_oracle_pins as pins

GOLDEN = pins.os.path.join(pins.os.path.dirname(pins.__file__), "golden")


def _fails(fn, *args):
    try:
        with np.errstate(all="ignore"):
            fn(*args)
    except (AssertionError, FloatingPointError, IndexError, ValueError):
        return True
    return False


def test_dropped_scale_is_caught(monkeypatch):
    def no_scale(q, K, V, scale):
        if K.shape[0] == 0:
            return np.zeros(V.shape[1])
        s = K @ q
        w = np.exp(s - s.max())
        return (w @ V) / w.sum()
    monkeypatch.setattr(oa, "softmax_attention", no_scale)
    assert _fails(pins.test_two_token_closed_form)
    assert _fails(pins.test_identity_table_equals_library_dense_attention)


def test_missing_max_subtraction_is_caught(monkeypatch):
    def no_max(q, K, V, scale):
        if K.shape[0] == 0:
            return np.zeros(V.shape[1])
        w = np.exp(scale * (K @ q))
        return (w @ V) / w.sum()
    monkeypatch.setattr(oa, "softmax_attention", no_max)
    assert _fails(pins.test_huge_scores_do_not_overflow_and_pick_the_argmax)


def test_transposed_operand_is_caught(monkeypatch):
    def uses_k_for_values(q, K, V, scale):
        if K.shape[0] == 0:
            return np.zeros(V.shape[1])
        s = scale * (K @ q)
        w = np.exp(s - s.max())
        return (w @ K) / w.sum()
    monkeypatch.setattr(oa, "softmax_attention", uses_k_for_values)
    assert _fails(pins.test_two_token_closed_form)
    assert _fails(pins.test_identity_table_equals_library_dense_attention)


def test_wrong_gqa_mapping_is_caught(monkeypatch):
    real = oa.gather_tokens

    def interleaved(pool, table, positions, B, kv_head):
        # plants h % H_kv: callers pass h // G, so remap back through G = 4
        return real(pool, table, positions, B, (kv_head * 4) % pool.shape[1] if pool.shape[1] > 1 else 0)
    monkeypatch.setattr(oa, "gather_tokens", interleaved)
    assert _fails(pins.test_identity_table_equals_library_dense_attention)
    assert _fails(pins.test_gqa_mapping_and_mha_special_case)


def test_wrong_offset_is_caught(monkeypatch):
    def off_by_one(table, position, B):
        return int(table[position // B]), (position + 1) % B
    monkeypatch.setattr(op, "translate", off_by_one)
    monkeypatch.setattr(oa, "translate", off_by_one)
    assert _fails(pins.test_address_translation_worked_example, GOLDEN)
    assert _fails(pins.test_identity_table_equals_library_dense_attention)


def test_merge_without_rescale_is_caught(monkeypatch):
    def naive(parts):
        parts = list(parts)
        num = sum(Z * np.asarray(o) for _, Z, o in parts)
        den = sum(Z for _, Z, _ in parts)
        return max(p[0] for p in parts), den, num / den
    monkeypatch.setattr(oa, "merge", naive)
    assert _fails(pins.test_merge_worked_example, GOLDEN)
    assert _fails(pins.test_split_partitions_match_single_pass)


def test_copy_on_write_in_place_is_caught(monkeypatch):
    def no_cow(self, seq_id):
        table = self.tables[seq_id]
        pos = self.lengths[seq_id]
        if pos % self.block_size == 0:
            table.append(self._take())
        self.lengths[seq_id] = pos + 1
        return op.flat_slot(table, pos, self.block_size)
    monkeypatch.setattr(op.BlockManager, "append_slot", no_cow)
    assert _fails(pins.test_copy_on_write_worked_example, GOLDEN)


@pytest.mark.parametrize("bad", ["ceil_minus_one", "floor"])
def test_wrong_block_count_is_caught(monkeypatch, bad):
    f = (lambda T, B: T // B) if bad == "floor" else (lambda T, B: max(0, -(-T // B) - 1))
    monkeypatch.setattr(op, "blocks_needed", f)
    assert _fails(pins.test_address_translation_worked_example, GOLDEN)
