"""The guard-and-repeat checker of test_gpu_guards.py, shown on the CPU to catch what it
is there to catch: a write one byte past an output, a write into the padding between
the rows of a strided output, a write past the workspace, an element left unwritten,
a result that changes between runs, and an input that a call modifies."""
import pytest
import torch

from guards import run_twice


def test_clean_call_passes():
    def call(ar):
        y = ar.out("y", 5, 24, torch.float32, ld=32)
        y.copy_(torch.arange(120, dtype=torch.float32).view(5, 24))
        ws = ar.workspace(1024)
        ws[256:].fill_(7)
    run_twice("clean", [], call, "cpu", status=lambda ws: int(ws[:4].view(torch.int32)[0]))


@pytest.mark.parametrize("fault,match", [
    ("past_end", "written outside 'y'"),
    ("row_padding", "written outside 'y'"),
    ("before_start", "written outside 'y'"),
    ("past_workspace", "written outside 'workspace'"),
    ("unwritten", "differs between two runs"),
    ("changing", "differs between two runs"),
    ("input", "an input changed"),
    ("status", "status word set"),
])
def test_planted_faults_are_caught(fault, match):
    x = torch.ones(8)
    runs = []

    def call(ar):
        runs.append(1)
        y = ar.out("y", 5, 24, torch.float32, ld=32)
        base = ar.bufs[-1][1]
        ws = ar.workspace(512)
        wsfull = ar.bufs[-1][1]
        y.copy_(torch.arange(120, dtype=torch.float32).view(5, 24))
        if fault == "past_end":
            base[4096 + 5 * 32 * 4] ^= 1
        elif fault == "row_padding":
            base[4096 + 24 * 4 + 3] ^= 1
        elif fault == "before_start":
            base[4095] ^= 1
        elif fault == "past_workspace":
            wsfull[4096 + 512] ^= 1
        elif fault == "unwritten":  # element (3, 0) keeps the run's random bytes
            o = 4096 + 3 * 32 * 4
            base[o:o + 4] = ar.bufs[0][2][o:o + 4]
        elif fault == "changing":
            y[1, 1] = float(len(runs))
        elif fault == "input":
            x[3] = 2.0
        elif fault == "status":
            ws[0] = 1

    with pytest.raises(AssertionError, match=match):
        run_twice(fault, [x], call, "cpu", status=lambda w: int(w[:4].view(torch.int32)[0]))
