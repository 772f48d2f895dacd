"""A CPU model of kda_chunk_fwd's segmented path (kda_api.cu): sequences whose
chunk records exceed the workspace cap run in segments over two record
buffers, each segment's prep (and exact) kernel on a low-priority stream and
its chain kernel on a high-priority one.  The model replays the host's enqueue
order (stream_model.py's event rules, random durations) and checks that:

* segment i's prep and exact kernels write buffer i % 2 only after the chain of
  segment i - 2 has read it;
* segment i's chain starts after its prep and exact kernels end, and after the
  chain of segment i - 1 (the carried state);
* the caller's later work follows every kernel of the call, and two calls on
  different streams never overlap on the shared workspace.

The launch-completion event that places segment i's chain CTAs before segment
i + 1's prep CTAs is a best effort (it may fire early, or only when the chain
ends): it orders for speed only, so the checks must hold for any firing time,
and the model fires it anywhere up to the chain's end.
Planted mistakes (each ordering wait taken out) must each break a check.
"""
import random

import pytest

from stream_model import overlap, simulate


def enqueue_call(nseg, skip=(), ops=None, call=0, caller="s"):
    ops = [] if ops is None else ops

    def add(stream, kind, arg=None):
        ops.append((caller if stream == "s" else stream, kind, arg))

    if "done" not in skip:
        add("s", "wait", "done")
    add("s", "record", "fork")
    add("lo", "wait", "fork")
    add("hi", "wait", "fork")
    for i in range(nseg):
        buf = i & 1
        if i >= 2 and "prep_after_chain" not in skip:
            add("lo", "wait", f"chain_done{buf}")
        if i >= 1:
            add("lo", "wait", "chain_go")
        add("lo", "op", ("prep", call, i, buf))
        add("lo", "op", ("exact", call, i, buf))
        add("lo", "record", f"prep_done{buf}")
        if "chain_after_prep" not in skip:
            add("hi", "wait", f"prep_done{buf}")
        add("hi", "record_start", "chain_go")
        add("hi", "op", ("chain", call, i, buf))
        add("hi", "record", f"chain_done{buf}")
    if "join" not in skip:
        add("s", "wait", f"chain_done{(nseg - 1) & 1}")
    add("s", "record", "done")
    add("s", "op", ("after", call, None, None))
    return ops


def violations(spans):
    bad = []
    by = {}
    for (what, call, i, buf), s, e, stream in spans:
        by[(what, call, i)] = (s, e, buf)
    calls = sorted({k[1] for k in by})
    for c in calls:
        n = max(k[2] for k in by if k[1] == c and k[2] is not None) + 1
        for i in range(n):
            p, x, ch = by[("prep", c, i)], by[("exact", c, i)], by[("chain", c, i)]
            if ch[0] < x[1] or ch[0] < p[1]:
                bad.append(f"call {c}: chain {i} started before its records were complete")
            if i >= 1 and ch[0] < by[("chain", c, i - 1)][1]:
                bad.append(f"call {c}: chain {i} started before chain {i - 1} ended")
            if i >= 2:
                old = by[("chain", c, i - 2)]
                if overlap(p, old) or overlap(x, old) or p[0] < old[0]:
                    bad.append(f"call {c}: segment {i} rewrote buffer {i & 1} under chain {i - 2}")
        after = by[("after", c, None)]
        for k, v in by.items():
            if k[1] == c and k[0] != "after" and v[1] > after[0] + 1e-12:
                bad.append(f"call {c}: {k[0]} {k[2]} still running when the caller's next work starts")
    # calls share the workspace: no kernel of one overlaps a kernel of another
    ks = [(k, v) for k, v in by.items() if k[0] in ("prep", "exact", "chain")]
    for a in range(len(ks)):
        for b in range(a + 1, len(ks)):
            (ka, va), (kb, vb) = ks[a], ks[b]
            if ka[1] != kb[1] and overlap(va, vb):
                bad.append(f"{ka} and {kb} of different calls overlap on the workspace")
    return bad


@pytest.mark.parametrize("nseg", [1, 2, 3, 6])
def test_segments_hold_under_random_durations(nseg):
    rng = random.Random(nseg)
    for _ in range(300):
        assert violations(simulate(enqueue_call(nseg), rng)) == []


@pytest.mark.parametrize("second_stream", ["s", "s2"])
def test_back_to_back_calls(second_stream):
    rng = random.Random(5)
    for _ in range(300):
        ops = enqueue_call(4, call=0)
        enqueue_call(3, ops=ops, call=1, caller=second_stream)
        assert violations(simulate(ops, rng)) == []


@pytest.mark.parametrize("mistake", ["prep_after_chain", "chain_after_prep", "join", "done"])
def test_each_wait_is_needed(mistake):
    rng = random.Random(13)
    found = False
    for _ in range(3000):
        ops = enqueue_call(4, skip=(mistake,), call=0)
        enqueue_call(4, skip=(mistake,), ops=ops, call=1, caller="s2")
        if violations(simulate(ops, rng)):
            found = True
            break
    assert found, mistake
