"""Failure detection without faulting the GPU: an allocator that refuses memory, a host wait
that runs past SOUP_WAIT_TIMEOUT_MS, and an in-kernel barrier wait that runs out (a barrier
nothing arrives on, through the library's own wait code).  Each error comes back as its status
code and the model (or the next model) keeps working."""
import ctypes
import math
import os

import pytest
import torch

import synth
from layer_streamed_nf4_lut_b200 import _lib
from layer_streamed_nf4_lut_b200._lib import SoupError, lib
from layer_streamed_nf4_lut_b200.model import make_config
from tests.gpu_util import Pair

pytestmark = pytest.mark.gpu


class FailingAllocator:
    """Allocates through torch's caching allocator; the k-th request (1-based) returns NULL."""

    def __init__(self, fail_at):
        self.fail_at, self.calls, self.live = fail_at, 0, set()

        def _alloc(nbytes, user):
            self.calls += 1
            if self.calls == self.fail_at:
                return None
            p = torch.cuda.caching_allocator_alloc(int(nbytes), 0)
            self.live.add(p)
            return p

        def _free(p, user):
            assert p in self.live, "freed a pointer the allocator never handed out"
            self.live.discard(p)
            torch.cuda.caching_allocator_delete(int(p))

        self._a, self._f = _lib.ALLOC_FN(_alloc), _lib.FREE_FN(_free)
        self.struct = _lib.Allocator(self._a, self._f, None)


@pytest.mark.parametrize("fail_at", [1, 2, 7, 40])
def test_allocator_returning_null_gives_oom_and_frees_everything(fail_at):
    cfg = make_config(dict(synth.TINY), "streamed", 2, 64)
    al = FailingAllocator(fail_at)
    h = ctypes.c_void_p()
    st = lib.soup_model_create(ctypes.byref(cfg), ctypes.byref(al.struct), ctypes.byref(h))
    assert st == -3, st  # SOUP_ERR_OOM
    assert al.calls == fail_at and not al.live  # every successful allocation was handed back
    # the next model (with an allocator that works) is fine
    ok = FailingAllocator(-1)
    assert lib.soup_model_create(ctypes.byref(cfg), ctypes.byref(ok.struct), ctypes.byref(h)) == 0
    assert ok.calls > fail_at and ok.live
    assert lib.soup_model_destroy(h) == 0
    assert not ok.live


def test_host_wait_timeout_then_next_step_succeeds(monkeypatch):
    p = Pair(dict(synth.TINY), seed=81, modes=("streamed",), want_oracle=False)
    try:
        gm = p.models["streamed"]
        ids = torch.from_numpy(synth.token_batch(p.cfg, 82)).cuda()
        want = gm.step(ids, apply_optimizer=False)
        torch.cuda.synchronize()
        # keep the stream busy for ~0.5 s ahead of the step, and bound the host wait at 1 ms
        torch.cuda._sleep(1_000_000_000)
        monkeypatch.setenv("SOUP_WAIT_TIMEOUT_MS", "1")
        with pytest.raises(SoupError) as ei:
            gm.step(ids, apply_optimizer=False)
        assert ei.value.status == -5  # SOUP_ERR_TIMEOUT
        monkeypatch.delenv("SOUP_WAIT_TIMEOUT_MS")
        torch.cuda.synchronize()
        assert gm.step(ids, apply_optimizer=False) == want
    finally:
        p.close()


def test_in_kernel_wait_runs_out_then_model_stays_usable():
    p = Pair(dict(synth.TINY), seed=83, modes=("resident",), want_oracle=False)
    try:
        gm = p.models["resident"]
        ids = torch.from_numpy(synth.token_batch(p.cfg, 84)).cuda()
        want = gm.step(ids, apply_optimizer=False)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        assert lib.soup_selftest_bounded_wait(gm.h, 2000, stream) == 0
        with pytest.raises(SoupError) as ei:
            gm.check_device()
        assert ei.value.status == -5  # the wait's error word -> SOUP_ERR_TIMEOUT
        gm.check_device()  # reported once, then cleared
        # a timed-out wait surfaces through the step too
        assert lib.soup_selftest_bounded_wait(gm.h, 1000, stream) == 0
        with pytest.raises(SoupError) as ei:
            gm.step(ids, apply_optimizer=False)
        assert ei.value.status == -5
        loss = gm.step(ids, apply_optimizer=False)
        assert math.isfinite(loss) and loss == want
        assert lib.soup_selftest_bounded_wait(gm.h, 0, stream) == -1  # limit out of range
    finally:
        p.close()
