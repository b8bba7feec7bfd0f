"""The fused kernel's mbarrier protocol, run as a discrete-event model (tests/tc_protocol_model.py).

Random unit sizes (including one-tile units) and random completion delays, for the ring depths
of both head dimensions and both schedules (groups on alternate tiles, the kernel's; groups on
column halves of every tile): no deadlock, no stale parity wait, no data hazard. Planted protocol
mistakes must each be caught: a QK^T that does not wait for the PV two tiles back, a PV-done
barrier with the wrong arrival count, and a producer that waits for the V stage's use before the
previous one.
"""
import random

import pytest

from tc_protocol_model import Protocol, random_plan


@pytest.mark.parametrize("schedule", ["split_single_issuer", "split_dephase", "smem_p", "group_issuers",
                                      "alternate", "split"])
@pytest.mark.parametrize("nk,nv", [(3, 2), (4, 4)])  # d = 128 and d = 64 ring depths
@pytest.mark.parametrize("route_in_kernel", [False, True])  # keep bits from the routing pass, or routed in place
def test_protocol_has_no_deadlock_stale_wait_or_hazard(nk, nv, route_in_kernel, schedule):
    rng = random.Random(nk * 10 + nv)
    for k in range(150):
        Protocol(random_plan(rng), seed=k, nk=nk, nv=nv, route_in_kernel=route_in_kernel, schedule=schedule).run()


@pytest.mark.parametrize("schedule,mutation", [
    ("split", "qk_skips_pvdone"), ("split", "pvdone_count_1"), ("split", "vempty_one_back"),
    ("alternate", "qk_skips_pvdone"), ("alternate", "alt_pvdone_count_2"), ("alternate", "vempty_one_back"),
    ("group_issuers", "qk_skips_pvdone"), ("group_issuers", "alt_pvdone_count_2"),
    ("group_issuers", "vempty_one_back"),
    ("smem_p", "qk_skips_sfree"), ("smem_p", "p_skips_pvdone"), ("smem_p", "vempty_one_back"),
    ("split_dephase", "qk_skips_sfree"), ("split_dephase", "p_skips_pvdone"), ("split_dephase", "vempty_one_back"),
    ("split_single_issuer", "vempty_one_back"),
])
def test_planted_protocol_mistakes_are_caught(schedule, mutation):
    rng = random.Random(5)
    caught = 0
    for k in range(150):
        try:
            Protocol(random_plan(rng), seed=k, mutation=mutation, schedule=schedule).run()
        except AssertionError:
            caught += 1
    assert caught > 0
