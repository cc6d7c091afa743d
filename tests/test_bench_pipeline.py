"""The benchmark's serving-pipeline schedule on CPU: the order in which
run_pipelined issues batch fronts (Stage I / append + auto-split) and backs
(Stage II), recorded by a fake workload."""
import bench


class Recorder:
    def __init__(self):
        self.calls = []

    def set_inputs(self, i):
        self.calls.append(("in", i))

    def front(self, k, main, serial=False):
        self.calls.append(("front", k, serial))

    def back(self, k, main):
        self.calls.append(("back", k))


def test_pipeline_issues_next_front_before_this_back_and_drains():
    r = Recorder()
    bench.run_pipelined(r, None, 4)
    assert r.calls == [("in", 0), ("front", 0, False),
                       ("in", 1), ("front", 1, False), ("back", 0),
                       ("in", 2), ("front", 2, False), ("back", 1),
                       ("in", 3), ("front", 3, False), ("back", 2),
                       ("back", 3)]


def test_serial_mode_runs_each_batch_whole_on_one_stream():
    r = Recorder()
    bench.run_pipelined(r, None, 3, serial=True)
    assert r.calls == [("in", 0), ("front", 0, True), ("back", 0),
                       ("in", 1), ("front", 1, True), ("back", 1),
                       ("in", 2), ("front", 2, True), ("back", 2)]


def test_every_batch_has_one_front_and_one_back():
    for n in (1, 2, 7):
        r = Recorder()
        bench.run_pipelined(r, None, n)
        fronts = [c[1] for c in r.calls if c[0] == "front"]
        backs = [c[1] for c in r.calls if c[0] == "back"]
        assert fronts == list(range(n)) and backs == list(range(n))
        # a batch's back always comes after its front
        pos = {c: i for i, c in enumerate(r.calls)}
        for k in range(n):
            assert pos[("back", k)] > pos[("front", k, False)]
