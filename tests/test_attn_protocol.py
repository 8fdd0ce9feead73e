"""The attention kernel's mbarrier protocol, checked on the CPU through a
discrete-event model of its warp roles (tests/attn_protocol_model.py): random
item structures (empty, single-step and long items, partial last steps) under
random completion delays and interleavings."""
import pytest

from attn_protocol_model import run_schedules


def test_protocol_has_no_deadlock_early_wait_or_early_reuse():
    """Every role finishes; each ring and record slot is reused only after its
    previous user is done; every parity wait except the epilogue's names its
    phase exactly."""
    run_schedules(300, seed=2026, check_epilogue=False)


def test_epilogue_wait_names_its_item():
    """With one O-complete barrier per item parity, the epilogue's parity wait
    succeeds on exactly its own item's phase, under every schedule."""
    run_schedules(600, seed=2026, check_epilogue=True)


def test_single_o_complete_barrier_is_caught():
    """The model tells the two designs apart: with a single O-complete barrier
    advancing once per item, some schedule lets an epilogue whose item starts
    right after the previous item's last step pass its wait one phase early."""
    with pytest.raises(AssertionError, match="o_full0"):
        run_schedules(300, seed=2026, check_epilogue=True, single_o_full=True)
