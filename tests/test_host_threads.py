"""Host-side planning from several threads, and the static workspace's size
(CPU only: the metadata builder and the split planner need no device).

The ABI promises that different handles may be used from different host
threads at once. The pieces of shared host state are the split override
(per calling thread) and the per-device caches of the launchers; these tests
drive two threads through metadata builds and split plans at the same time
(ctypes releases the interpreter lock for the duration of each C call) and
check every result against the same work done on one thread.
"""
import threading

import pytest

from segment_causal_masked_b200 import sca
from segment_causal_masked_b200 import workloads as W


def _plans(problem, sms_list, override):
    sca.set_split_override(override)
    try:
        md = sca.build_for(problem)
        return [sca.attn_plan_for_sms(md, problem.heads, sms) for sms in sms_list]
    finally:
        sca.set_split_override(0)


def test_split_override_is_per_thread():
    """An override set on one thread does not reach another thread's plans."""
    p = W.small_session(heads=4)
    md = sca.build_for(p)
    auto = sca.attn_plan_for_sms(md, p.heads, 148)
    seen = {}
    ready, done = threading.Event(), threading.Event()

    def other():
        sca.set_split_override(7)
        ready.set()
        done.wait(10)
        seen["other"] = sca.attn_plan_for_sms(sca.build_for(p), p.heads, 148)
        sca.set_split_override(0)

    t = threading.Thread(target=other)
    t.start()
    assert ready.wait(10)
    seen["main"] = sca.attn_plan_for_sms(md, p.heads, 148)
    done.set()
    t.join(10)
    assert seen["main"] == auto
    assert seen["other"]["chunks"] == 7


def test_two_threads_build_and_plan_at_once():
    problems = [W.session_480p_single_turn(), W.small_packed(seed=21, n_segments=14),
                W.with_history(W.small_session(heads=4), 1), W.small_session(heads=4)]
    sms_list = [132, 148, 160]
    serial = [_plans(p, sms_list, ov) for p, ov in zip(problems, (0, 3, 0, 5))]
    results, errors = {}, []

    def worker(i):
        try:
            for _ in range(3):
                results.setdefault(i, []).append(_plans(problems[i], sms_list, (0, 3, 0, 5)[i]))
        except Exception as e:  # pragma: no cover - reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(problems))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(120)
    assert not errors, errors
    for i in range(len(problems)):
        assert results[i] == [serial[i]] * 3


@pytest.mark.parametrize("make", [
    W.session_480p_single_turn, W.session_480p_long,
    lambda: W.with_history(W.session_480p_long(), 4),
    lambda: W.with_random_blocks(W.session_480p_long(), 0.25, 25, group=2),
    lambda: W.with_random_blocks(W.with_history(W.session_480p_long(), 4), 0.25, 11),
], ids=["single-turn", "long-session", "long-window4", "long-blocks25", "long-window4-blocks25"])
def test_static_workspace_holds_the_480p_split_plans_on_148_sms(make):
    """The allocation-free entry point's fixed array is sized for the 480p
    layouts' automatic split plans on a 148-SM B200 (other SM counts may
    plan larger splits; those calls run unsplit)."""
    p = make()
    plan = sca.attn_plan_for_sms(sca.build_for(p), p.heads, 148)
    assert plan["chunks"] > 1
    assert 0 < plan["workspace_bytes"] <= sca.STATIC_WORKSPACE_BYTES
