"""A model of prism_layer_step_host's stream and event ordering, checked on the CPU.

This is not the library code: it restates, as a sequence of stream operations,
what layer.cu enqueues for one host-buffer step.
- The h2d stream uploads V, hhat, Q, K and dO.
- The compute stream runs the forward and the backward.
- The d2h stream downloads O, dQ, dK and dV.
- Events join the streams. A wait takes the most recent record of its event at
  the time of the call, and a never-recorded event counts as complete, as in CUDA.

Several steps are issued back to back, each with its own data, and a random
scheduler runs the streams' operations in any order their FIFOs and waits allow.
Every read must find the data of its own step: a compute stage reading an input,
or a download reading an output. That holds in the blocked layout, where the
inputs are released after the permutes that read them, and in the raster layout,
where they are released only at the end of the step.
"""
import random

import pytest


class Model:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.streams = {"h2d": [], "compute": [], "d2h": []}
        self.buf = {}                 # device buffer -> step whose data it holds
        self.done = set()             # completed operation ids
        self.events = {}              # event name -> op id of its latest record (None: never recorded)
        self.n = 0

    def _op(self, stream, kind, **kw):
        self.n += 1
        self.streams[stream].append(dict(id=self.n, kind=kind, **kw))
        return self.n

    # what a host thread enqueues
    def record(self, stream, event):
        # the record completes once the stream reaches it
        self.events[event] = self._op(stream, "record")

    def wait(self, stream, event):
        self._op(stream, "wait", on=self.events.get(event))

    def write(self, stream, name, step):
        self._op(stream, "write", name=name, step=step)

    def read(self, stream, name, step):
        self._op(stream, "read", name=name, step=step)

    def run(self):
        while any(self.streams.values()):
            ready = [s for s, q in self.streams.items()
                     if q and (q[0]["kind"] != "wait" or q[0]["on"] is None or q[0]["on"] in self.done)]
            assert ready, "deadlock"
            op = self.streams[self.rng.choice(ready)].pop(0)
            if op["kind"] == "write":
                self.buf[op["name"]] = op["step"]
            elif op["kind"] == "read":
                assert self.buf.get(op["name"]) == op["step"], (op, self.buf.get(op["name"]))
            self.done.add(op["id"])


def step_host(m, step, raster, bwd=True, release_early=False):
    """The enqueue order of one prism_layer_step_host call (layer.cu).
    release_early plants a mistake: the blocked layout's release of the inputs
    recorded before the permute of Q and K instead of after it."""
    m.record("d2h", f"prev_d2h{step}")
    m.wait("h2d", "inputs_read")
    for name in ("V", "hhat"):
        m.write("h2d", name, step)
    m.record("h2d", f"vh{step}")
    for name in ("Q", "K"):
        m.write("h2d", name, step)
    m.record("h2d", f"qk{step}")
    if bwd:
        m.wait("h2d", "do_read")
        m.write("h2d", "dO", step)
        m.record("h2d", f"do{step}")
    # forward
    m.wait("compute", f"vh{step}")
    m.read("compute", "V", step)                      # zone indicator
    m.read("compute", "hhat", step)
    if raster:
        m.wait("compute", f"qk{step}")
        for name in ("Q", "K"):                      # pooled scores through the permutation
            m.read("compute", name, step)
        m.wait("compute", f"prev_d2h{step}")
        for name in ("Q", "K", "V"):                 # attention on the raster operands
            m.read("compute", name, step)
        m.write("compute", "O", step)
    else:
        m.read("compute", "V", step)                  # permute V
        m.wait("compute", f"qk{step}")
        if release_early:
            m.record("compute", "inputs_read")
        m.read("compute", "Q", step)                  # permute Q, K
        m.read("compute", "K", step)
        if not release_early:
            m.record("compute", "inputs_read")
        m.wait("compute", f"prev_d2h{step}")
        m.write("compute", "O", step)                 # unpermute O
    m.record("compute", f"o{step}")
    m.wait("d2h", f"o{step}")
    m.read("d2h", "O", step)
    if bwd:
        m.wait("compute", f"do{step}")
        if raster:
            for name in ("Q", "K", "V", "dO"):
                m.read("compute", name, step)
        else:
            m.read("compute", "dO", step)             # permute dO
            m.record("compute", "do_read")
        for name in ("dQ", "dK", "dV"):
            m.write("compute", name, step)
            m.record("compute", f"{name}{step}")
        for name in ("dQ", "dK", "dV"):
            m.wait("d2h", f"{name}{step}")
            m.read("d2h", name, step)
    if raster:                                        # the inputs are read until here
        m.record("compute", "inputs_read")
        m.record("compute", "do_read")


@pytest.mark.parametrize("raster", [False, True])
@pytest.mark.parametrize("bwd", [True, False])
def test_back_to_back_steps_read_their_own_data(raster, bwd):
    for seed in range(400):
        m = Model(seed)
        for step in range(4):
            step_host(m, step, raster, bwd)
        m.run()


def test_model_catches_an_input_released_too_early():
    """Releasing Q, K, V and hhat before the permute of Q and K has read them lets
    the next step's upload overwrite a live input."""
    with pytest.raises(AssertionError):
        for seed in range(400):
            m = Model(seed)
            for step in range(4):
                step_host(m, step, raster=False, release_early=True)
            m.run()


def test_model_catches_a_download_overwritten(monkeypatch):
    """Without the wait for the previous step's downloads, O of the next step can
    overwrite O before the previous step's download has read it."""
    orig = Model.record

    def record(self, stream, event):
        if event.startswith("prev_d2h"):
            self.events[event] = None                 # the record dropped: the wait passes at once
            return
        orig(self, stream, event)

    monkeypatch.setattr(Model, "record", record)
    with pytest.raises(AssertionError):
        for seed in range(400):
            m = Model(seed)
            for step in range(4):
                step_host(m, step, raster=False)
            m.run()


def test_model_catches_raster_inputs_never_released(monkeypatch):
    """With raster operands the attention reads Q, K, V and dO until the end of the
    backward: without that release the next step's uploads overwrite them."""
    orig = Model.record

    def record(self, stream, event):
        if event in ("inputs_read", "do_read"):
            return                                    # never recorded: the next uploads do not wait
        orig(self, stream, event)

    monkeypatch.setattr(Model, "record", record)
    with pytest.raises(AssertionError):
        for seed in range(400):
            m = Model(seed)
            for step in range(4):
                step_host(m, step, raster=True)
            m.run()
