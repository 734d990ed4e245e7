"""The bounded pipeline waits, exercised without any fault: a test hook makes the decode
step's producer withhold one tile (no copy issued, no arrival), so the consumers' waits run
out after a short limit; the kernel must report LA_DEVERR_TIMEOUT, return promptly, and leave
the context usable for the next, normal call."""
import time

import pytest
import torch

from gated_deltanet_recurrent_la_b200 import lastate as L
from gated_deltanet_recurrent_la_b200 import workloads as W
from gpu_helpers import check_step_against_oracle, gpu_step

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _hooks_reset():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    L.la_debug_set_wait_limit_us(0)
    L.la_debug_withhold_step_tile(-1)


def test_withheld_tile_times_out_and_the_context_recovers():
    inp = W.step_inputs(B=8, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, n_slots=16, slot_map="perm", seed=71)
    check_step_against_oracle(inp)  # warm: the kernel is loaded, the call is correct
    L.la_debug_set_wait_limit_us(2000)
    L.la_debug_withhold_step_tile(0)
    t0 = time.perf_counter()
    _, _, err = gpu_step(inp)
    elapsed = time.perf_counter() - t0
    assert err & L.DEVERR_TIMEOUT, f"error word {err}: the withheld arrival must be reported"
    assert elapsed < 0.5, f"the expired waits must end the kernel promptly ({elapsed:.3f} s)"
    # the hook is one-shot and the context is healthy: the next step is complete and correct
    L.la_debug_set_wait_limit_us(0)
    check_step_against_oracle(inp)


def test_hooks_are_inert_when_not_reached():
    """A withheld tile index the first CTA never reaches changes nothing."""
    inp = W.step_inputs(B=8, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, n_slots=16, slot_map="perm", seed=72)
    L.la_debug_set_wait_limit_us(2000)
    L.la_debug_withhold_step_tile(1 << 30)
    check_step_against_oracle(inp)
