"""bench.py's end-to-end measurement (host copies inside the timed region) run against a
simulated device: streams, events and three engines (host-to-device copies, compute,
device-to-host copies) on a virtual clock.  CPU only.

Every operation logs the buffers it reads and writes with its simulated start and end.  The
tests check that no two operations touch one buffer at overlapping times when either writes it,
that such operations run in program order (no step reads inputs that a later copy has already
replaced, no copy-out reads results that a later step has already overwritten), and that the
pipelined form overlaps the copies of neighbouring steps with the compute.
"""

import contextlib
import types

import pytest

import bench

H2D_GBS = D2H_GBS = 50.0   # simulated copy engines, GB/s
FWD_MS, BWD_MS = 0.5, 1.1


class FakeTensor:
    _next = 0

    def __init__(self, nbytes, where, numel=None):
        FakeTensor._next += 1
        self.id = FakeTensor._next
        self.nbytes = nbytes
        self.where = where               # "host", "pinned" or "dev"
        self._numel = numel if numel is not None else nbytes // 2

    def numel(self):
        return self._numel

    def element_size(self):
        return self.nbytes // self._numel

    def pin_memory(self):
        return FakeTensor(self.nbytes, "pinned", self._numel)

    def __getitem__(self, _):
        return FakeTensor(0, self.where, 1)

    def copy_(self, src, non_blocking=False):
        assert non_blocking
        if src.where == "pinned" and self.where == "dev":
            engine, gbs = "h2d", H2D_GBS
        elif src.where == "dev" and self.where == "pinned":
            engine, gbs = "d2h", D2H_GBS
        else:
            raise AssertionError("copy between unexpected memories")
        SIM.op(engine, src.nbytes / (gbs * 1e9) * 1e3, reads=[src], writes=[self])
        return self


class Sim:
    def __init__(self):
        self.reset()

    def reset(self):
        self.engines = {"h2d": 0.0, "d2h": 0.0, "sm": 0.0}
        self.log = []            # (seq, start, end, reads, writes, engine)
        self.default = FakeStream()
        self.current = self.default

    def op(self, engine, ms, reads=(), writes=()):
        s = self.current
        start = max(s.t, self.engines[engine])
        end = start + ms
        s.t = end
        self.engines[engine] = end
        self.log.append((len(self.log), start, end, [t.id for t in reads], [t.id for t in writes], engine))


class FakeStream:
    def __init__(self, device=None):
        self.t = 0.0

    def wait_event(self, ev):
        if ev.t is not None:
            self.t = max(self.t, ev.t)


class FakeEvent:
    def __init__(self, enable_timing=False):
        self.t = None

    def record(self, stream=None):
        self.t = (stream or SIM.current).t

    def elapsed_time(self, other):
        return other.t - self.t


SIM = Sim()


def _make_torch(stream_fails=False):
    def synchronize(device=None):
        t = max([SIM.default.t] + list(SIM.engines.values()))
        SIM.default.t = t

    @contextlib.contextmanager
    def stream_ctx(s):
        prev, SIM.current = SIM.current, s
        try:
            yield
        finally:
            SIM.current = prev

    def make_stream(device=None):
        if stream_fails:
            raise RuntimeError("no streams here")
        return FakeStream(device)

    cuda = types.SimpleNamespace(Event=FakeEvent, Stream=make_stream, stream=stream_ctx, synchronize=synchronize)

    def empty_like(x, device=None, dtype=None):
        return FakeTensor(x.nbytes, "dev" if device is not None or x.where == "dev" else x.where, x.numel())

    def empty(shape, dtype=None, device=None):
        n = 1
        for s in (shape if isinstance(shape, tuple) else (shape,)):
            n *= s
        size = 4 if dtype == "f32" else 1
        return FakeTensor(n * size, "dev" if device is not None else "host", n)

    return types.SimpleNamespace(cuda=cuda, empty_like=empty_like, empty=empty, float32="f32", uint8="u8")


class FakeFA:
    @staticmethod
    def bwd_workspace_size(B, H, N, d):
        return 1 << 20

    @staticmethod
    def forward(q, k, v, scale, causal, window, out=None, lse=None):
        SIM.op("sm", FWD_MS, reads=[q, k, v], writes=[out, lse])
        return out, lse

    @staticmethod
    def backward(q, k, v, o, lse, do, scale, causal, window, grads=None, workspace=None):
        SIM.op("sm", BWD_MS, reads=[q, k, v, o, lse, do], writes=list(grads) + [workspace])
        return grads


def _run(stream_fails=False, steps=10):
    SIM.reset()
    FakeTensor._next = 0
    wl = types.SimpleNamespace(B=2, H=32, N=4096, d=128, scale=0.088, causal=True, window=0)
    nbytes = wl.B * wl.H * wl.N * wl.d * 2
    q_h, k_h, v_h, do_h = (FakeTensor(nbytes, "host") for _ in range(4))
    torch = _make_torch(stream_fails)
    res = bench.measure_e2e(FakeFA, torch, wl, "dev", SIM.default, q_h, k_h, v_h, do_h, True, steps, 1e12, 1)
    return res, nbytes


def _check_no_hazards():
    """Operations sharing a buffer, one of them writing it, neither overlap in time nor run out
    of program order."""
    for i, (si, a0, a1, ri, wi, _) in enumerate(SIM.log):
        for sj, b0, b1, rj, wj, _ in SIM.log[i + 1:]:
            shared = (set(wi) & (set(rj) | set(wj))) | (set(ri) & set(wj))
            if shared:
                assert a1 <= b0 + 1e-12, ("overlap or reorder on a buffer", si, sj, a0, a1, b0, b1)


def test_pipelined_e2e_overlaps_copies_with_compute():
    res, nbytes = _run()
    assert res["mode"].startswith("pipelined")
    h2d_ms = 4 * nbytes / (H2D_GBS * 1e9) * 1e3
    d2h_ms = (4 * nbytes + 2 * 32 * 4096 * 4) / (D2H_GBS * 1e9) * 1e3
    serial_ms = h2d_ms + FWD_MS + BWD_MS + d2h_ms
    bound = max(h2d_ms, d2h_ms, FWD_MS + BWD_MS)
    assert res["ms_per_step"] <= 1.15 * bound, (res["ms_per_step"], bound)
    assert res["ms_per_step"] < 0.7 * serial_ms
    assert res["h2d_bytes_per_step"] == 4 * nbytes
    _check_no_hazards()


def test_every_step_copies_in_and_out():
    """Four inputs in (Q, K, V, dO) and five results out (O, L, dQ, dK, dV) per step, for the
    timed steps and the two warm-up steps."""
    steps = 10
    _run(steps=steps)
    engines = [e[5] for e in SIM.log]
    assert engines.count("h2d") == 4 * (steps + 2)
    assert engines.count("d2h") == 5 * (steps + 2)
    assert engines.count("sm") == 2 * (steps + 2)


def test_serial_fallback_is_measured_and_named():
    res, nbytes = _run(stream_fails=True)
    assert res["mode"].startswith("serial")
    h2d_ms = 4 * nbytes / (H2D_GBS * 1e9) * 1e3
    assert res["ms_per_step"] >= h2d_ms + FWD_MS + BWD_MS
    _check_no_hazards()


def test_hazard_check_catches_a_missing_wait(monkeypatch):
    """Plant the bug the waits prevent: the copy streams wait for nothing, so a copy-in may
    overwrite inputs a step still reads and a copy-out may read results not yet written.  The
    hazard check must fail."""
    orig = FakeStream.wait_event

    def copy_streams_do_not_wait(self, ev):
        if self is SIM.default:
            orig(self, ev)

    monkeypatch.setattr(FakeStream, "wait_event", copy_streams_do_not_wait)
    _run()
    with pytest.raises(AssertionError):
        _check_no_hazards()
