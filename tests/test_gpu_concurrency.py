"""Calls from several host threads at once, each on its own stream: the
launchers' one-time setup and the host pipeline's queues are shared per
device, and every call must still give the bits of a sequential run. ctypes
releases the interpreter lock around foreign calls, so the threads really
enter the library concurrently."""
import threading

import pytest
import torch

import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def test_device_and_host_calls_from_four_threads():
    w = wi.Workload("case", 1, (3, 10, 13), 6)
    gq_h, gk_h = wi.gammas(w.heads)
    gq, gk = gq_h.cuda(), gk_h.cuda()
    inputs = [wi.packed_qkv(w.batch, w.seq_len, w.heads, seed=60 + k) for k in range(8)]
    refs = []
    for x in inputs:
        d = x.cuda()
        refs.append(wan.dit_attn(d, w.grid, w.heads, gq, gk).cpu())
    torch.cuda.synchronize()

    results, errors = {}, []

    def worker(t):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):  # copies and allocations of this thread on its stream
                for rep in range(3):
                    for k in range(t, len(inputs), 4):
                        if (k + rep) % 2 == 0:
                            d = inputs[k].cuda()
                            out = wan.dit_attn(d, w.grid, w.heads, gq, gk, stream=s)
                        else:
                            out = wan.dit_attn_host(inputs[k].pin_memory(), w.grid, w.heads, gq, gk, stream=s)
                        s.synchronize()
                        results[(t, rep, k)] = out.cpu()
        except Exception as e:  # reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(t,)) for t in range(4)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    assert wan.device_error() == 0
    assert len(results) == 3 * len(inputs)
    for (t, rep, k), out in results.items():
        assert torch.equal(out.view(torch.int16), refs[k].view(torch.int16)), (t, rep, k)
