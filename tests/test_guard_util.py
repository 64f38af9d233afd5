"""The canary guard bands of the parity tests catch writes outside an output
(checked here on the CPU by planting one, as an overrunning kernel would)."""
import pytest
import torch

from parity_util import GUARD, _GUARDED, check_guards, guarded_empty


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.int16, torch.float32])
@pytest.mark.parametrize("where", ["before", "after"])
def test_planted_overrun_is_caught(dtype, where):
    t = guarded_empty((7, 16), dtype, "cpu")
    assert t.data_ptr() % 16 == 0
    t.zero_()  # writing the output itself is fine
    buf = _GUARDED[-1][0]
    buf[GUARD - 1 if where == "before" else GUARD + 7 * 16] = 0
    with pytest.raises(AssertionError, match="write outside an output"):
        check_guards()


def test_clean_outputs_pass():
    a = guarded_empty((3, 5), torch.bfloat16, "cpu")
    b = guarded_empty((2, 8), torch.float32, "cpu")
    a.fill_(1.0)
    b.fill_(-2.0)
    check_guards()
