"""The end-to-end pipeline's ordering, checked without a device: recording
fakes stand in for CUDA streams and events, and the happens-before relation
they build (stream order plus event waits) must order every reuse of a
buffer slot after the work that last read it, while leaving the input copy
of one step free to overlap the result copy of the step before."""
import contextlib

import bench


class FakeEvent:
    def __init__(self):
        self.node = None          # the last node of the stream when recorded

    def record(self, stream):
        self.node = stream.nodes[-1] if stream.nodes else None


class FakeStream:
    def __init__(self, graph, name):
        self.graph, self.name, self.nodes = graph, name, []

    def add(self, label):
        node = self.graph.new_node(label, self)
        if self.nodes:
            self.graph.edge(self.nodes[-1], node)   # stream order
        self.nodes.append(node)
        return node

    def wait_event(self, ev):
        node = self.add(("wait", self.name))
        if ev.node is not None:                     # an unrecorded event is no wait
            self.graph.edge(ev.node, node)


class Graph:
    def __init__(self):
        self.succ, self.labels, self.current = {}, {}, None

    def new_node(self, label, stream):
        n = len(self.labels)
        self.labels[n] = label
        self.succ[n] = []
        return n

    def edge(self, a, b):
        self.succ[a].append(b)

    def before(self, a, b):
        seen, todo = set(), [a]
        while todo:
            x = todo.pop()
            if x == b:
                return True
            if x in seen:
                continue
            seen.add(x)
            todo.extend(self.succ[x])
        return False


class FakeWorkload:
    """Records each phase on the current fake stream, with its step index."""

    def __init__(self, graph):
        self.g = graph
        self.count = {"h2d": 0, "comp": 0, "d2h": 0}
        self.node = {}

    def _op(self, kind, j):
        i = self.count[kind]
        self.count[kind] += 1
        assert i % 2 == j
        self.node[(kind, i)] = self.g.current.add((kind, i))

    def e2e_h2d(self, j):
        self._op("h2d", j)

    def e2e_compute(self, j):
        self._op("comp", j)

    def e2e_d2h(self, j):
        self._op("d2h", j)


def test_pipeline_orders_slot_reuse_and_overlaps_copies():
    g = Graph()
    names = iter(["h2d", "compute", "d2h"])

    @contextlib.contextmanager
    def on_stream(s):
        prev, g.current = g.current, s
        try:
            yield
        finally:
            g.current = prev

    wl = FakeWorkload(g)
    pipe = bench.E2EPipeline(wl, None, new_stream=lambda: FakeStream(g, next(names)), new_event=FakeEvent,
                             on_stream=on_stream)
    n = 9
    for i in range(n):
        pipe.step(i)
    node = wl.node
    for i in range(n):
        assert g.before(node[("h2d", i)], node[("comp", i)])       # compute after its input
        assert g.before(node[("comp", i)], node[("d2h", i)])       # result copy after compute
        if i >= 2:
            # slot reuse: the input copy after the compute that last read the
            # slot's input, the compute after the copy that last read its D
            assert g.before(node[("comp", i - 2)], node[("h2d", i)])
            assert g.before(node[("d2h", i - 2)], node[("comp", i)])
        if i >= 1:
            # copies in and out of consecutive steps are not serialised
            assert not g.before(node[("d2h", i - 1)], node[("h2d", i)])
            assert not g.before(node[("h2d", i)], node[("d2h", i - 1)])
