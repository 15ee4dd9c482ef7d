"""First calls on a device, each in a fresh process: two host threads racing the first
launches (the per-device kernel set-up runs once, under a lock), and decode and varlen
calls made under CUDA stream capture after the device's first call (their workspace comes
from the library's stream-ordered pool, so the capture holds the allocation and the
free)."""
import os
import subprocess
import sys

import pytest

from fa_testlib import has_b200

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_THREADS = r"""
import sys, threading
sys.path.insert(0, sys.argv[1])
import torch
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import make_qkv, make_grad_out

torch.cuda.set_device(0)
cases = [make_qkv(1, 4, 700, 700, 128, torch.bfloat16, 100 * t, device="cuda") for t in range(2)]
decs = [make_qkv(2, 8, 1, 3000, 64, torch.float16, 100 * t + 50, device="cuda") for t in range(2)]
gos = [make_grad_out(1, 4, 700, 128, torch.bfloat16, 100 * t + 9, device="cuda") for t in range(2)]
torch.cuda.synchronize()
gate = threading.Barrier(2)
res = [None, None]

def work(t):
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q, k, v = cases[t]
        gate.wait()   # both threads enter the library's first launches together
        o, lse = binding.attention(q, k, v, causal=True, out_dtype=torch.bfloat16)
        od, ld = binding.attention(*decs[t])
        g = binding.attention_backward(q, k, v, o, lse, gos[t], causal=True)
        s.synchronize()
        res[t] = (o, lse, od, ld) + tuple(g)

th = [threading.Thread(target=work, args=(t,)) for t in range(2)]
for x in th: x.start()
for x in th: x.join()
assert all(r is not None for r in res), "a thread failed"
for t in range(2):   # the same calls again, one thread: bitwise the same outputs
    q, k, v = cases[t]
    o, lse = binding.attention(q, k, v, causal=True, out_dtype=torch.bfloat16)
    od, ld = binding.attention(*decs[t])
    dq, dk, dv = binding.attention_backward(q, k, v, o, lse, gos[t], causal=True)
    torch.cuda.synchronize()
    got = res[t][:4] + res[t][5:]
    for a, b in zip(got, (o, lse, od, ld, dk, dv)):
        assert torch.equal(a, b)
    # dQ is summed in arrival order: equal within fp32 rounding, not bitwise
    assert (res[t][4].float() - dq.float()).abs().max().item() <= 1e-2
assert binding.fa_device_status(clear=True) == 0
print("OK")
"""

_CAPTURE = r"""
import sys
sys.path.insert(0, sys.argv[1])
import torch
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import make_qkv, randn

torch.cuda.set_device(0)
shapes = [(4, 8, 5000), (16, 32, 9000)]   # the second needs more workspace than the first
data = [make_qkv(B, H, 1, N, 128, torch.bfloat16, 31 + B, device="cuda") for B, H, N in shapes]
outs = [(torch.empty((B, H, 1, 128), device="cuda"), torch.empty((B, H, 1), device="cuda"))
        for B, H, _ in shapes]
# The device's first call, outside capture (it sets the device up).
qp, kp, vp = make_qkv(1, 2, 300, 300, 128, torch.bfloat16, 5, device="cuda")
binding.attention(qp, kp, vp, causal=True)
# a packed batch for a varlen call under capture
lens = [300, 5, 700]
cu = torch.tensor([0, 300, 305, 1005], dtype=torch.int32, device="cuda")
vq, vk, vv = (randn((1005, 2, 64), 77 + i, torch.float16, device="cuda") for i in range(3))
vo = torch.empty((1005, 2, 64), device="cuda")
vl = torch.empty((1005, 2), device="cuda")
torch.cuda.synchronize()
s = torch.cuda.Stream()
graph = torch.cuda.CUDAGraph()
with torch.cuda.graph(graph, stream=s):
    for (q, k, v), (o, l), (B, H, N) in zip(data, outs, shapes):
        rc = binding.fa_fwd_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   l.data_ptr(), B, H, N, 128, 0.088, s.cuda_stream,
                                   binding.FA_BF16, binding.FA_F32, 0)
        assert rc == binding.FA_OK, (rc, binding.fa_get_last_cuda_error())
    rc = binding.fa_fwd_varlen(vq.data_ptr(), vk.data_ptr(), vv.data_ptr(), vo.data_ptr(),
                               vl.data_ptr(), cu.data_ptr(), cu.data_ptr(), 3, 2, 1005, 1005,
                               700, 700, 64, 0.125, 1, s.cuda_stream, binding.FA_F16,
                               binding.FA_F32)
    assert rc == binding.FA_OK, (rc, binding.fa_get_last_cuda_error())
for _ in range(2):
    for o, l in outs + [(vo, vl)]:
        o.fill_(float("nan")); l.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    for (q, k, v), (o, l) in zip(data, outs):
        o2, l2 = binding.attention(q, k, v, scale=0.088)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(l, l2)
    o2, l2 = binding.varlen_attention(vq, vk, vv, cu, cu, 700, 700, causal=True, scale=0.125)
    torch.cuda.synchronize()
    assert torch.equal(vo, o2) and torch.equal(vl, l2)
del graph
assert binding.fa_device_status(clear=True) == 0
binding.fa_release_workspace()
print("OK")
"""


def _run(script):
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")
    r = subprocess.run([sys.executable, "-c", script, ROOT], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr


def test_two_threads_race_the_first_launches():
    _run(_THREADS)


def test_workspace_calls_under_stream_capture():
    _run(_CAPTURE)
