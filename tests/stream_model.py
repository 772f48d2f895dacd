"""A tiny model of CUDA stream and event ordering for protocol tests (CPU only).

Operations are replayed in host program order as (stream, kind, arg):
* ("op", payload): work on the stream, with a random duration;
* ("record", event): the event captures everything enqueued on the stream so far
  (waits included);
* ("wait", event): the stream's later work starts after the work captured by the
  event's most recent record made before this wait (no-op if never recorded);
* ("record_start", event): a launch-completion event attached to the stream's
  next op.  The runtime fires it once every CTA of that kernel has begun, but
  only as a best effort: a kernel ordered after it may start earlier, or wait
  for the whole kernel.  So the model fires it at a random time anywhere before
  the op's end, even before the op starts: it guarantees no ordering.
"""


def simulate(ops, rng):
    """[(payload, start, end, stream)] for every "op" under the rules above."""
    stream_end, stream_ready, record_time, pending_start = {}, {}, {}, {}
    spans = []
    for stream, kind, arg in ops:
        t = stream_end.get(stream, 0.0)
        ready = max(t, stream_ready.get(stream, 0.0))
        if kind == "record":
            record_time[arg] = ready
        elif kind == "record_start":
            pending_start.setdefault(stream, []).append(arg)
        elif kind == "wait":
            if arg in record_time:
                stream_ready[stream] = max(stream_ready.get(stream, 0.0), record_time[arg])
        else:
            start = ready
            end = start + rng.uniform(0.1, 3.0)
            for ev in pending_start.pop(stream, []):
                record_time[ev] = rng.uniform(0.0, end)
            stream_end[stream] = end
            spans.append((arg, start, end, stream))
    return spans


def overlap(a, b):
    return a[0] < b[1] and b[0] < a[1]
