"""The library's calls inside a CUDA graph.

Every entry point enqueues on the stream it is given, never synchronises and
allocates nothing in the call itself, so a whole decoder block (GroupNorm
statistics -> normalise + SiLU -> convolution with the residual) and the
backward pass can be captured once and replayed.  The replays must reproduce
the eager results bit for bit (the weight gradient's fp32 atomics excepted:
within the parity tolerance of the eager result).
"""
import pytest
import torch

import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from parity import assert_close

pytestmark = pytest.mark.gpu

CREP = c3.TPAD_CAUSAL_REPLICATE


def _block_inputs():
    N, D, H, W, C = 1, 4, 24, 40, 128
    x = si.tensor((N, D, H, W, C), 51, 0, 1.0, torch.bfloat16, "cuda")
    gamma = (si.tensor((C,), 51, 1, 0.2, torch.float32, "cuda") + 1.0).to(torch.bfloat16)
    beta = si.tensor((C,), 51, 2, 0.2, torch.bfloat16, "cuda")
    w = si.tensor((C, 3, 3, 3, C), 51, 1, (27 * C) ** -0.5, torch.bfloat16, "cuda")
    bias = si.tensor((C,), 51, 2, 0.1, torch.bfloat16, "cuda")
    return x, gamma, beta, w, bias


def test_decoder_block_graph_replays_bitwise():
    x, gamma, beta, w, bias = _block_inputs()
    stats = torch.empty((1, 32, 2), dtype=torch.float64, device="cuda")
    h = torch.empty_like(x)
    y = torch.empty_like(x)

    def block(stream):
        c3.groupnorm_stats(x, 32, 1e-6, False, stats, stream)
        c3.groupnorm_silu(x, stats, gamma, beta, h, 32, False, True, stream)
        c3.conv3d_fwd(h, w, bias, x, y, (1, 1, 1), (0, 1, 1), CREP, stream=stream)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        block(s)                                 # eager (also sets the kernels' attributes)
    torch.cuda.synchronize()
    ref = y.clone()
    y.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        block(torch.cuda.current_stream())
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert c3.poll_status() == c3.Status.OK
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_backward_graph_replays():
    x, _, _, w, _ = _block_inputs()
    dy = si.tensor(x.shape, 52, 5, 1.0, torch.bfloat16, "cuda")
    k = (3, 3, 3)
    dx = torch.empty_like(x)
    dw = torch.empty_like(w)
    db = torch.empty((w.shape[0],), dtype=torch.bfloat16, device="cuda")
    N, D, H, W, C = x.shape
    ws_d = torch.empty(c3.bwd_data_workspace_bytes(N, C, D, H, W, C, k, (0, 1, 1), CREP),
                       dtype=torch.uint8, device="cuda")
    ws_w = torch.empty(c3.bwd_weight_workspace_bytes(C, C, k), dtype=torch.uint8, device="cuda")

    def backward(stream):
        h = c3._stream_handle(stream)
        assert c3.conv3d_bwd_data_ptr(dy.data_ptr(), w.data_ptr(), dx.data_ptr(), N, C, D, H, W, C,
                                      k, (1, 1, 1), (0, 1, 1), CREP, c3.BF16, ws_d.data_ptr(),
                                      ws_d.numel(), h) == c3.Status.OK
        assert c3.conv3d_bwd_weight_ptr(x.data_ptr(), dy.data_ptr(), dw.data_ptr(), db.data_ptr(),
                                        N, C, D, H, W, C, k, (1, 1, 1), (0, 1, 1), CREP, c3.BF16,
                                        ws_w.data_ptr(), ws_w.numel(), h) == c3.Status.OK

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        backward(s)
    torch.cuda.synchronize()
    ref_dx, ref_dw, ref_db = dx.clone(), dw.clone(), db.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        backward(torch.cuda.current_stream())
    for _ in range(2):
        dx.zero_(); dw.zero_(); db.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert c3.poll_status() == c3.Status.OK
        assert torch.equal(dx.view(torch.int16), ref_dx.view(torch.int16))
        assert_close(dw.double().cpu().numpy(), ref_dw.double().cpu().numpy(), "dw replay")
        assert_close(db.double().cpu().numpy(), ref_db.double().cpu().numpy(), "dbias replay")
