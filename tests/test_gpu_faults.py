"""Device fault reporting on the GPU: check=True raises on a bad slot, and the
fault word's read-and-clear (kvq_get_error, one atomic exchange on the device)
never loses a bit that a kernel on another stream raises while other callers
are reading the word."""
import threading
import time

import pytest
import torch

import kv_cache_quantize_b200 as kvq

pytestmark = pytest.mark.gpu


def _bad_slot_call():
    """One-row compress call whose slot lies one past the cache (16 slots)."""
    dev = torch.device("cuda")
    x = torch.zeros((1, 128), dtype=torch.bfloat16, device=dev)
    bad = torch.tensor([16], dtype=torch.int32, device=dev)
    cache = torch.zeros((1, 16, 1, 224), dtype=torch.uint8, device=dev)
    return x, bad, cache


def test_check_flag_raises_on_a_bad_slot():
    x, bad, cache = _bad_slot_call()
    kvq.get_error()
    with pytest.raises(kvq.KvqFault) as e:
        kvq.kv_compress_epilog(x, bad, cache, 0, check=True)
    assert e.value.bits == kvq.FAULT_SLOT_RANGE
    assert kvq.get_error() == 0                      # the check consumed the bit
    assert int(cache.sum()) == 0                     # the row was skipped
    good = torch.tensor([3], dtype=torch.int32, device=x.device)
    kvq.kv_compress_epilog(x, good, cache, 0, check=True)


def test_fault_bit_is_never_lost_between_get_error_calls():
    """Stream s1 raises the slot bit once per round; a second thread reads and
    clears the word on stream s2 in a tight loop.  Each round's bit must reach
    exactly one reader: the polling thread, or the raiser's own get_error."""
    x, bad, cache = _bad_slot_call()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    kvq.get_error()
    seen_by_poller = threading.Event()
    stop = threading.Event()
    polls = [0]

    def poll():
        while not stop.is_set():
            if kvq.get_error(s2) & kvq.FAULT_SLOT_RANGE:
                seen_by_poller.set()
            polls[0] += 1

    th = threading.Thread(target=poll, daemon=True)
    th.start()
    by_raiser = by_poller = lost = 0
    try:
        for _ in range(400):
            seen_by_poller.clear()
            kvq.kv_compress_epilog(x, bad, cache, 0, stream=s1)
            s1.synchronize()
            deadline = time.monotonic() + 2.0
            while True:
                if kvq.get_error(s1) & kvq.FAULT_SLOT_RANGE:
                    by_raiser += 1
                    break
                if seen_by_poller.is_set():
                    by_poller += 1
                    break
                if time.monotonic() > deadline:
                    lost += 1
                    break
    finally:
        stop.set()
        th.join()
    print(f"rounds seen by the raiser {by_raiser}, by the poller {by_poller}, polls {polls[0]}")
    assert lost == 0
    assert kvq.get_error() == 0
