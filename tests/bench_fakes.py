"""Runs bench.py's main() on a machine without a GPU, with torch.cuda's
streams, events and graphs and the library's layer calls replaced by fakes
that only count and order calls.  It checks the benchmark's control flow and
its JSON line (keys, step counts, launch counts, timing labels), never a
number: the fakes measure nothing.

    python tests/bench_fakes.py <bench.py arguments>

prints bench.py's JSON line, then a line "CALLS <layer calls executed>".
"""
import contextlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

_device = torch.device
_capturing = []
_calls = {"n": 0}


def _run_or_capture(fn):
    if _capturing:
        _capturing[-1].nodes.append(fn)
    else:
        fn()


class Event:
    clock = 0.0

    def __init__(self, enable_timing=False, external=False):
        self.when = None

    def _stamp(self):
        Event.clock += 0.01
        self.when = Event.clock

    def record(self, stream=None):
        _run_or_capture(self._stamp)

    def elapsed_time(self, other):
        assert self.when is not None and other.when is not None, "an event was never recorded"
        return other.when - self.when

    def synchronize(self):
        pass


class Stream:
    def __init__(self, *a, **k):
        pass

    def synchronize(self):
        pass

    def wait_stream(self, other):
        pass


class CUDAGraph:
    def __init__(self):
        self.nodes = None

    def replay(self):
        assert self.nodes is not None, "replay before capture"
        for fn in self.nodes:
            fn()


@contextlib.contextmanager
def graph(g, stream=None):
    g.nodes = []
    _capturing.append(g)
    try:
        yield
    finally:
        _capturing.pop()


def _device_or_cpu(kind, index=None):
    if kind == "cuda":
        return _device("cpu")
    return _device(kind) if index is None else _device(kind, index)


class Layer:
    def __init__(self, *a, **k):
        self.handle = 1

    def last_error(self):
        return 0

    def close(self):
        pass


def _layer_call(*a, **k):
    def bump():
        _calls["n"] += 1
    _run_or_capture(bump)
    return 0


class _NoClocks:
    def __init__(self, *a):
        pass

    def start(self):
        pass

    def stop(self):
        return {"sm_mhz": 0.0, "sm_max_mhz": 0.0, "reasons": [], "samples": 0}


def main(argv):
    torch.cuda.set_device = lambda *a: None
    torch.cuda.Stream = Stream
    torch.cuda.Event = Event
    torch.cuda.CUDAGraph = CUDAGraph
    torch.cuda.graph = graph
    torch.cuda.synchronize = lambda *a: None
    torch.cuda.stream = lambda s: contextlib.nullcontext()
    torch.cuda.memory_allocated = lambda *a: 0
    torch.device = _device_or_cpu
    from hybrid_linear_attention_arl2_b200 import arl2
    arl2.load_library = lambda *a, **k: None
    arl2.HybridLayer = arl2.HybridBlock = arl2.KVLayer = Layer
    for name in ("arl2_frame_query", "arl2_frame_commit", "arl2_block_query", "arl2_block_commit",
                 "arl2_kv_query", "arl2_kv_commit", "arl2_token_query", "arl2_token_commit"):
        setattr(arl2, name, _layer_call)
    import bench
    bench.ClockSampler = _NoClocks
    sys.argv = ["bench.py"] + argv
    bench.main()
    print("CALLS", _calls["n"], flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
