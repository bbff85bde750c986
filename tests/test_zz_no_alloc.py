"""nvfp4_linear_noalloc: the workspace-free, allocation-free variant of nvfp4_linear.

The pages have no counterpart (it is a deployment variant).  Two consecutive calls
on the library's one per-device buffer must each give exactly the result of
nvfp4_linear with a caller workspace, and after the first call on the device (which
may load the buffer's module) further calls must not change the device's free
memory.  Collected last on purpose (file name), and independent of the tests before
it: it sets the GEMM kernel choice itself and restores it.
"""
import pytest
import torch

import synth
import block_scaled_precision_act_b200 as bsp

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def automatic_kernel_choice():
    old = bsp.bsp_testing_set_gemm_kernel(0)
    yield
    bsp.bsp_testing_set_gemm_kernel(old)


def problem(M, N, K, seed, with_bias):
    a = synth.bf16_normal((M, K), 1.0, seed, 0.01, 20.0).cuda()
    w = synth.bf16_normal((N, K), 0.02, seed + 1).cuda()
    bias = synth.bf16_normal((N,), 0.5, seed + 2).cuda() if with_bias else None
    ga = bsp.nvfp4_global_scale(a)
    gw = bsp.nvfp4_global_scale(w)
    wc, wsf = bsp.nvfp4_quantize_act(w, gw, layout=bsp.SF_MMA)
    return a, ga, wc, wsf, gw, bias


def test_noalloc_matches_linear_on_two_consecutive_calls():
    p1 = problem(4096, 3072, 3072, 500, True)       # the attention projection at 1 MP
    p2 = problem(200, 136, 320, 510, False)         # ragged, different size
    outs, refs = [], []
    for a, ga, wc, wsf, gw, bias in (p1, p2):
        y = torch.empty((a.shape[0], wc.shape[0]), dtype=torch.bfloat16, device="cuda")
        outs.append(bsp.nvfp4_linear_noalloc(a, ga, wc, wsf, gw, out=y, bias=bias))
    for a, ga, wc, wsf, gw, bias in (p1, p2):
        refs.append(bsp.nvfp4_linear(a, ga, wc, wsf, gw, bias=bias))
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    for y, r in zip(outs, refs):
        assert torch.equal(y, r)


def test_noalloc_leaves_free_memory_unchanged():
    a, ga, wc, wsf, gw, bias = problem(1024, 768, 1024, 520, True)
    ys = [torch.empty((1024, 768), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    bsp.nvfp4_linear_noalloc(a, ga, wc, wsf, gw, out=ys[0], bias=bias)   # first use on device
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    bsp.nvfp4_linear_noalloc(a, ga, wc, wsf, gw, out=ys[1], bias=bias)
    bsp.nvfp4_linear_noalloc(a, ga, wc, wsf, gw, out=ys[2], bias=bias)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert bsp.bsp_last_device_status() == 0
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def test_noalloc_rejects_oversize_problem():
    """A problem whose workspace exceeds the fixed buffer is refused before any launch
    (real buffers of the full size: no call here hands the library an address it does
    not own)."""
    K, N = 3072, 256
    rows = bsp.nvfp4_linear_noalloc_max_bytes() // (K // 2) + 1
    assert bsp.nvfp4_linear_workspace_bytes(rows, K) > bsp.nvfp4_linear_noalloc_max_bytes()
    a = torch.zeros((rows, K), dtype=torch.bfloat16, device="cuda")
    _, ga, wc, wsf, gw, _ = problem(128, N, K, 530, False)
    y = torch.zeros((rows, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bsp.BSPError) as err:
        bsp.nvfp4_linear_noalloc(a, ga, wc, wsf, gw, out=y)
    assert err.value.status == -2
    torch.cuda.synchronize()
    assert not torch.any(y)                              # nothing was launched
    assert bsp.bsp_last_device_status() == 0


CAPTURE_FIRST = r"""
import sys, torch
sys.path.insert(0, {root!r})
sys.path.insert(0, {tests!r})
import synth
import block_scaled_precision_act_b200 as bsp
a = synth.bf16_normal((256, 512), 1.0, 540).cuda()
w = synth.bf16_normal((384, 512), 0.02, 541).cuda()
ga, gw = bsp.nvfp4_global_scale(a), bsp.nvfp4_global_scale(w)
wc, wsf = bsp.nvfp4_quantize_act(w, gw)
ref = bsp.nvfp4_linear(a, ga, wc, wsf, gw)        # every other path initialised first
torch.cuda.synchronize()
y = torch.empty_like(ref)
stream = torch.cuda.Stream()
graph = torch.cuda.CUDAGraph()
first = "captured"
try:
    with torch.cuda.graph(graph, stream=stream):
        bsp.nvfp4_linear_noalloc(a, ga, wc, wsf, gw, out=y)
except Exception as e:                            # the lookup may be refused in a capture
    first = "refused: " + type(e).__name__
torch.cuda.synchronize()
del graph
y2 = bsp.nvfp4_linear_noalloc(a, ga, wc, wsf, gw, out=torch.empty_like(ref))  # retried
c, s = bsp.nvfp4_quantize_act(a, ga)              # no stale CUDA error left behind
torch.cuda.synchronize()
assert torch.equal(y2, ref), "noalloc after the capture differs from nvfp4_linear"
assert bsp.bsp_last_device_status() == 0
print("OK", first)
"""


def test_noalloc_first_call_inside_a_capture_does_not_poison_later_calls():
    """The buffer's address is looked up on the first call on a device, which the header
    asks callers to make outside stream capture.  If a caller makes it inside one and the
    lookup is refused, that call fails, but the failure must not stay cached nor leave a
    pending CUDA error: the next call outside the capture succeeds and equals
    nvfp4_linear, and the next unrelated library call returns OK.  Run in a fresh
    process, so that this really is the first call on the device."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = CAPTURE_FIRST.format(root=root, tests=os.path.join(root, "tests"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "OK" in r.stdout
