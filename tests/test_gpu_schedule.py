"""The benchmark's overlapped layer schedule (later weights' S and h on a
second stream beside the sweeps) writes exactly what the one-stream order
writes: every h, S, code and scale byte, over several back-to-back steps.
Needs a B200."""
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _layer():
    import workloads
    # a smaller layer of the 70B-shaped MLP's structure: two weights share one
    # calibration input, the third has its own
    s = 4000
    mats = [workloads.Matrix("gate", 1024, 2048, "gu", s + 1, 0.015, 0.001, 10.0),
            workloads.Matrix("up", 1024, 2048, "gu", s + 2, 0.015, 0.001, 10.0),
            workloads.Matrix("down", 2048, 1024, "down", s + 3, 0.015, 0.001, 10.0)]
    cal = {"gu": workloads.Calib("gu", 4096, 2048, 1.5, s + 41),
           "down": workloads.Calib("down", 4096, 1024, 1.5, s + 42)}
    return workloads.Workload("schedule_check", 448.0, mats, cal, [workloads.Run(-9, 6, True)])


def _poison(step):
    # what a sweep would read if it ran before its h or S were written
    for t in list(step.h.values()) + list(step.S.values()):
        t.fill_(float("nan"))
    for t in list(step.codes.values()) + list(step.scales.values()):
        t.fill_(0xAA)
    torch.cuda.synchronize()


def _run(step, n):
    for _ in range(n):
        step.run()
    torch.cuda.synchronize()
    return ({k: v.clone() for k, v in step.h.items()}, {k: v.clone() for k, v in step.S.items()},
            {k: v.clone() for k, v in step.codes.items()}, {k: v.clone() for k, v in step.scales.items()})


def test_overlapped_layer_matches_serial():
    import bench
    import block_scale_search_b200 as nv
    nv.lib()
    wl = _layer()
    Ws = {m.name: m.make(DEV) for m in wl.matrices}
    Xs = {k: c.make(DEV) for k, c in wl.calibs.items()}
    ser = _run(bench.Step(nv, wl, Ws, Xs, torch.device(DEV), serial=True), 1)
    step = bench.Step(nv, wl, Ws, Xs, torch.device(DEV), serial=False)
    _poison(step)
    for n in (1, 3):        # one step on poisoned buffers, then back-to-back steps
        ovl = _run(step, n)
        for a, b in zip(ser, ovl):
            assert a.keys() == b.keys()
            for k in a:
                assert torch.equal(a[k].view(torch.uint8), b[k].view(torch.uint8)), (n, k)
