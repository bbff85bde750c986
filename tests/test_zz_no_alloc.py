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
    K = 3072
    need_rows = bsp.nvfp4_linear_noalloc_max_bytes() // (K // 2) + 1
    assert bsp.nvfp4_linear_workspace_bytes(need_rows, K) > bsp.nvfp4_linear_noalloc_max_bytes()
    P = 1 << 20   # never dereferenced: the size check comes first
    st = bsp.lib().nvfp4_linear_noalloc(P, P, P, P, P, None, P, need_rows, 256, K, None)
    assert st == -2
