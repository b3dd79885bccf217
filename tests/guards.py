"""Guarded output buffers and the two-run comparison used by the out-of-bounds and race
tests (test_gpu_guards.py); device-agnostic so that test_guard_checker.py can show, on
the CPU, that a stray write and an unwritten element are both caught."""
import numpy as np

GUARD = 4096  # bytes on each side of a buffer; keeps the buffer 256-byte aligned


class Arena:
    """Buffers cut from allocations with random guard bytes around them."""

    def __init__(self, seed, device="cuda"):
        import torch
        self.torch = torch
        self.device = device
        self.gen = torch.Generator().manual_seed(seed)
        self.bufs = []     # (name, full, pattern, keep_mask)
        self.outs = {}     # name -> the view a call writes
        self.ws = None

    def _full(self, nbytes):
        torch = self.torch
        pattern = torch.randint(0, 256, (nbytes + 2 * GUARD,), dtype=torch.uint8,
                                generator=self.gen).to(self.device)
        return pattern.clone(), pattern

    def out(self, name, rows, cols, dtype, ld=None):
        """A [rows, cols] output with leading dimension ld (elements); the bytes of each
        row past `cols` must keep their pattern."""
        torch = self.torch
        ld = ld or cols
        es = torch.empty((), dtype=dtype).element_size()
        nbytes = rows * ld * es
        full, pattern = self._full(nbytes)
        keep = torch.ones(full.numel(), dtype=torch.bool, device=self.device)
        keep[GUARD:GUARD + nbytes].view(rows, ld * es)[:, :cols * es] = False
        view = full[GUARD:GUARD + nbytes].view(dtype).view(rows, ld)[:, :cols]
        self.bufs.append((name, full, pattern, keep))
        self.outs[name] = view
        return view

    def flat(self, name, nbytes, dtype):
        es = self.torch.empty((), dtype=dtype).element_size()
        return self.out(name, 1, nbytes // es, dtype)[0]

    def workspace(self, nbytes):
        """Status region zeroed, the rest random; only the guards are checked."""
        torch = self.torch
        nbytes = max(int(nbytes), 256)
        full, pattern = self._full(nbytes)
        full[GUARD:GUARD + 256] = 0
        pattern[GUARD:GUARD + 256] = 0
        keep = torch.ones(full.numel(), dtype=torch.bool, device=self.device)
        keep[GUARD:GUARD + nbytes] = False
        self.bufs.append(("workspace", full, pattern, keep))
        self.ws = full[GUARD:GUARD + nbytes]
        return self.ws

    def check_guards(self, what):
        for name, full, pattern, keep in self.bufs:
            bad = (full != pattern) & keep
            if bool(bad.any()):
                idx = bad.nonzero().flatten()
                first = int(idx[0]) - GUARD
                raise AssertionError(f"{what}: {int(idx.numel())} bytes written outside "
                                     f"'{name}', the first at offset {first} of the buffer")

    def output_bytes(self):
        return {k: v.contiguous().view(self.torch.uint8).cpu().numpy()
                for k, v in self.outs.items()}


def run_twice(what, inputs, call, device="cuda", status=None):
    """call(arena) writes into arena buffers. Checks the guards after each of two runs
    (the outputs start from different random bytes), the workspace status word
    (status(ws) -> int, when a workspace was used), that the inputs are unchanged and
    that the two runs wrote the same output bytes."""
    import torch
    before = [t.clone() for t in inputs]
    results = []
    for seed in (11, 12):
        arena = Arena(seed, device)
        call(arena)
        if device == "cuda":
            torch.cuda.synchronize()
        arena.check_guards(what)
        if arena.ws is not None and status is not None:
            assert status(arena.ws) == 0, f"{what}: status word set"
        results.append(arena.output_bytes())
    for t, b in zip(inputs, before):
        assert torch.equal(t, b), f"{what}: an input changed"
    for k in results[0]:
        a, b = results[0][k], results[1][k]
        if not np.array_equal(a, b):
            n = int((a != b).sum())
            raise AssertionError(f"{what}: '{k}' differs between two runs in {n} of {a.size} "
                                 f"bytes (unwritten elements or a race)")
