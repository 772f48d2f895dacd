"""A CPU model of kda_chunk_fwd_host's stream protocol (host_fwd.cu).

The host call enqueues, in program order, uploads on one copy stream, prefills
on the caller's stream and downloads on another copy stream, ordered by CUDA
events over two staging slots.  The model replays that enqueue order with the
runtime's event semantics (a wait orders its stream after the work captured by
the most recent record of the event made before the wait was enqueued; a wait
on an event never recorded is a no-op) and random durations, and checks that:

* piece i is computed after its upload and downloaded after its compute;
* no upload writes a slot's inputs while another piece's compute reads them;
* no compute writes a slot's output while another piece's download reads it;
* the computes run in piece order (each continues the previous one's state);
* work the caller enqueues on its stream after the call starts only once every
  copy of the call has ended; two back-to-back calls share the slots safely.

Planted mistakes (each wait taken out in turn) must each break a check.
"""
import random

import pytest

from stream_model import simulate


def enqueue_call(npieces, skip=(), ops=None, call=0, caller="s"):
    """The enqueue sequence of one kda_chunk_fwd_host call made on stream `caller`:
    (stream, kind, arg); "up" and "down" are the library's copy streams."""
    ops = [] if ops is None else ops

    def add(stream, kind, arg=None):
        ops.append((caller if stream == "s" else stream, kind, arg))

    if "done" not in skip:
        add("s", "wait", "done")
    add("s", "record", "fork")
    add("up", "wait", "fork")
    add("down", "wait", "fork")
    add("up", "op", ("h0", call, None, None))
    for i in range(npieces):
        b = i & 1
        if i >= 2 and "up_after_compute" not in skip:
            add("up", "wait", f"computed{b}")
        add("up", "op", ("upload", call, i, b))
        add("up", "record", f"uploaded{b}")
        add("s", "wait", f"uploaded{b}")
        if i >= 2 and "compute_after_download" not in skip:
            add("s", "wait", f"downloaded{b}")
        add("s", "op", ("compute", call, i, b))
        add("s", "record", f"computed{b}")
        if "download_after_compute" not in skip:
            add("down", "wait", f"computed{b}")
        add("down", "op", ("download", call, i, b))
        add("down", "record", f"downloaded{b}")
    add("s", "op", ("hT", call, None, None))
    add("up", "record", "uploaded0")
    add("down", "record", "downloaded0")
    if "join" not in skip:
        add("s", "wait", "uploaded0")
        add("s", "wait", "downloaded0")
    add("s", "record", "done")
    add("s", "op", ("after", call, None, None))  # the caller's next work on its stream
    return ops


def violations(spans):
    bad = []
    by = {}
    for (what, call, i, b), s, e, stream in spans:
        by[(what, call, i)] = (s, e, b)

    def overlap(x, y):
        return x[0] < y[1] and y[0] < x[1]

    calls = sorted({k[1] for k in by})
    for c in calls:
        n = max(k[2] for k in by if k[1] == c and k[2] is not None) + 1
        for i in range(n):
            up, cp, dn = by[("upload", c, i)], by[("compute", c, i)], by[("download", c, i)]
            if cp[0] < up[1]:
                bad.append(f"call {c}: compute {i} before its upload ended")
            if dn[0] < cp[1]:
                bad.append(f"call {c}: download {i} before its compute ended")
            if i > 0 and cp[0] < by[("compute", c, i - 1)][1]:
                bad.append(f"call {c}: compute {i} before compute {i - 1} ended")
        hT = by[("hT", c, None)]
        if hT[0] < by[("compute", c, n - 1)][1]:
            bad.append(f"call {c}: hT read before the last compute ended")
    ups = [(k, v) for k, v in by.items() if k[0] == "upload"]
    cps = [(k, v) for k, v in by.items() if k[0] == "compute"]
    dns = [(k, v) for k, v in by.items() if k[0] == "download"]
    for (ku, u) in ups:
        for (kc, c) in cps:
            if u[2] == c[2] and (ku[1], ku[2]) != (kc[1], kc[2]) and overlap(u, c):
                bad.append(f"upload {ku[1:]} overwrote slot {u[2]} while compute {kc[1:]} read it")
    for (kc, c) in cps:
        for (kd, d) in dns:
            if c[2] == d[2] and (kc[1], kc[2]) != (kd[1], kd[2]) and overlap(c, d):
                bad.append(f"compute {kc[1:]} wrote slot {c[2]} while download {kd[1:]} read it")
    # the caller's next work on its stream starts after every copy of the call
    for (what, call, i, b), s, e, stream in spans:
        if stream in ("up", "down") and e > by[("after", call, None)][0] + 1e-12:
            bad.append(f"call {call}: {what} {i} still running when the caller's next work starts")
    return bad


@pytest.mark.parametrize("npieces", [1, 2, 3, 7])
def test_protocol_holds_under_random_durations(npieces):
    rng = random.Random(npieces)
    for _ in range(300):
        ops = enqueue_call(npieces)
        assert violations(simulate(ops, rng)) == []


@pytest.mark.parametrize("second_stream", ["s", "s2"])
def test_back_to_back_calls_share_the_staging(second_stream):
    """Two calls enqueued one after the other, on the same caller stream or on two."""
    rng = random.Random(7)
    for _ in range(300):
        ops = enqueue_call(3, call=0)
        enqueue_call(4, ops=ops, call=1, caller=second_stream)
        assert violations(simulate(ops, rng)) == []


@pytest.mark.parametrize("mistake", ["up_after_compute", "compute_after_download", "download_after_compute",
                                     "join", "done"])
def test_each_wait_is_needed(mistake):
    """Without any one of the waits, some interleaving breaks a check."""
    rng = random.Random(11)
    found = False
    for _ in range(2000):
        ops = enqueue_call(4, skip=(mistake,), call=0)
        enqueue_call(4, skip=(mistake,), ops=ops, call=1, caller="s2")
        if violations(simulate(ops, rng)):
            found = True
            break
    assert found, mistake
