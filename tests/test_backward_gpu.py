"""GPU backward pass against the fp64 oracle's adjoints (parity tolerance:
max|err| <= 1e-2 max|ref|, relative L1 <= 2e-3)."""
import pytest
import torch

import oracle
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from parity import assert_close

pytestmark = pytest.mark.gpu

ZERO, CREP, CZERO = c3.TPAD_ZERO, c3.TPAD_CAUSAL_REPLICATE, c3.TPAD_CAUSAL_ZERO
TD = {"bf16": (torch.bfloat16, oracle.BF16), "f16": (torch.float16, oracle.F16)}


def grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed, dt, stride=(1, 1, 1)):
    td, od = TD[dt]
    fan = Cin * k[0] * k[1] * k[2]
    x = si.tensor((N, D, H, W, Cin), seed, 0, 1.0, td, "cuda")
    w = si.tensor((Cout, *k, Cin), seed, 1, fan ** -0.5, td, "cuda")
    out = oracle.output_shape(D, H, W, k, stride, pad, tpad)
    dy = si.tensor((N, *out, Cout), seed, 5, 1.0, td, "cuda")
    return x, w, dy, od


@pytest.fixture(params=["single", "swap"])
def variant(request, monkeypatch):
    monkeypatch.setenv("CONV3D_CTA_PAIR", "0")
    monkeypatch.setenv("CONV3D_SWAP", "1" if request.param == "swap" else "0")
    return request.param


DATA_CASES = [
    # N, Cin, D, H, W, Cout, kernel, pad, tpad, dtype
    (1, 64, 4, 10, 12, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16"),
    (2, 64, 3, 9, 13, 128, (3, 3, 3), (0, 1, 1), CZERO, "bf16"),
    (1, 32, 5, 8, 8, 48, (3, 3, 3), (1, 1, 1), ZERO, "f16"),
    (1, 64, 6, 7, 9, 64, (3, 3, 3), (0, 1, 1), ZERO, "bf16"),        # pt = 0: Do = D - 2
    (1, 128, 2, 16, 16, 64, (1, 1, 1), (0, 0, 0), ZERO, "bf16"),
    (1, 48, 3, 11, 10, 40, (2, 3, 3), (0, 0, 1), CREP, "bf16"),
    (1, 64, 1, 12, 12, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16"),       # single frame
    (3, 64, 4, 8, 10, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16"),        # body launch per sample
    (2, 128, 2, 9, 7, 64, (2, 3, 3), (0, 1, 1), CREP, "f16"),         # kt = 2, two samples
    (2, 64, 1, 8, 8, 128, (3, 3, 3), (0, 1, 1), CREP, "bf16"),        # single frame, two samples
    (1, 64, 3, 1, 1, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16"),         # 1x1 frames
    (1, 32, 2, 2, 300, 64, (3, 3, 3), (1, 1, 1), ZERO, "bf16"),       # rows longer than a tile
]


@pytest.mark.parametrize("case", DATA_CASES, ids=lambda c: "x".join(map(str, c[:6])) + f"-k{''.join(map(str, c[6]))}-t{c[8]}-{c[9]}")
def test_bwd_data_every_element(case, variant):
    N, Cin, D, H, W, Cout, k, pad, tpad, dt = case
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=300 + Cin, dt=dt)
    dx = c3.conv3d_bwd_data(dy, w, x.shape, pad, tpad)
    assert c3.poll_status() == c3.Status.OK
    ref, _, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, (1, 1, 1),
                                       pad, tpad)
    assert_close(dx.double().cpu().numpy(), ref, str(case))


def test_bwd_data_rejects_strides_and_cached_mode():
    x, w, dy, _ = grads_problem(1, 64, 4, 8, 8, 64, (3, 3, 3), (0, 1, 1), CREP, 1, "bf16",
                                stride=(2, 2, 2))
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    st = c3.conv3d_bwd_data_ptr(dy.data_ptr(), w.data_ptr(), x.data_ptr(), 1, 64, 4, 8, 8, 64,
                                (3, 3, 3), (2, 2, 2), (0, 1, 1), CREP, c3.BF16, ws.data_ptr(),
                                ws.numel(), 0)
    assert st == c3.Status.UNSUPPORTED


WEIGHT_CASES = [
    # N, Cin, D, H, W, Cout, kernel, stride, pad, tpad, dtype
    (1, 64, 4, 10, 12, 64, (3, 3, 3), (1, 1, 1), (0, 1, 1), CREP, "bf16"),
    (2, 128, 3, 9, 13, 256, (3, 3, 3), (1, 1, 1), (0, 1, 1), CZERO, "bf16"),
    (1, 32, 5, 8, 8, 48, (3, 3, 3), (1, 1, 1), (1, 1, 1), ZERO, "f16"),
    (1, 64, 5, 12, 12, 64, (3, 3, 3), (2, 2, 2), (0, 1, 1), CREP, "bf16"),   # strided
    (1, 256, 2, 16, 16, 320, (1, 1, 1), (1, 1, 1), (0, 0, 0), ZERO, "bf16"), # 2 co tiles, 1x1x1
    (1, 192, 3, 7, 9, 40, (2, 3, 3), (1, 1, 1), (0, 1, 1), CREP, "bf16"),    # partial blocks
    (1, 64, 6, 8, 8, 64, (3, 3, 3), (1, 1, 1), (3, 1, 1), ZERO, "bf16"),     # taps fully in padding
    (1, 128, 4, 9, 11, 96, (3, 3, 3), (1, 1, 1), (0, 1, 1), CZERO, "f16"),   # 18 entries per tap
    (1, 64, 3, 8, 8, 320, (1, 3, 3), (1, 1, 1), (0, 1, 1), ZERO, "bf16"),    # 3 co tiles of 128
    (2, 64, 1, 10, 12, 64, (3, 3, 3), (1, 1, 1), (0, 1, 1), CREP, "bf16"),   # single frame: taps equal
    (1, 128, 1, 9, 9, 96, (2, 3, 3), (1, 1, 1), (0, 1, 1), CREP, "f16"),     # single frame, kt = 2
    (1, 64, 3, 1, 1, 256, (3, 3, 3), (1, 1, 1), (0, 1, 1), CREP, "bf16"),    # 1x1 frames
    (1, 256, 2, 2, 300, 256, (3, 3, 3), (1, 1, 1), (1, 1, 1), ZERO, "bf16"), # rows longer than a chunk
]


@pytest.fixture(params=["plain", "pair", "swap"])
def wgrad_variant(request, monkeypatch):
    """The weight-gradient kernel's variants: one CTA, a CTA pair (256-channel output
    tiles only) and the swapped operand assignment (Cin % 64 == 0 only); where a
    variant does not apply the call falls back to the plain one."""
    monkeypatch.setenv("CONV3D_WGRAD_SWAP", "1" if request.param == "swap" else "0")
    monkeypatch.setenv("CONV3D_WGRAD_PAIR", "1" if request.param == "pair" else "0")
    return request.param


@pytest.mark.parametrize("case", WEIGHT_CASES, ids=lambda c: "x".join(map(str, c[:6])) + f"-k{''.join(map(str, c[6]))}-s{''.join(map(str, c[7]))}-t{c[9]}-{c[10]}")
def test_bwd_weight_every_element(case, wgrad_variant):
    N, Cin, D, H, W, Cout, k, stride, pad, tpad, dt = case
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=400 + Cin, dt=dt,
                                 stride=stride)
    dw, db = c3.conv3d_bwd_weight(x, dy, k, stride, pad, tpad)
    assert c3.poll_status() == c3.Status.OK
    _, ref_dw, ref_db = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, stride,
                                               pad, tpad)
    assert_close(dw.double().cpu().numpy(), ref_dw, "dw " + str(case))
    assert_close(db.double().cpu().numpy(), ref_db, "dbias " + str(case))


@pytest.mark.parametrize("side", ["beside", "after"])
@pytest.mark.parametrize("case", [WEIGHT_CASES[i] for i in (0, 1, 2, 4, 6, 8, 9)],
                         ids=lambda c: "x".join(map(str, c[:6])) + f"-t{c[9]}-{c[10]}")
def test_bwd_weight_bias_gradient_beside_and_after(case, side, monkeypatch):
    # The bias-gradient pass runs on the aux stream beside the weight-gradient
    # kernel (the default) or after it on the caller's stream
    # (CONV3D_WGRAD_DBIAS_SIDE=0); either way dbias is the oracle's sum over
    # every output pixel, and dw is unchanged.
    monkeypatch.setenv("CONV3D_WGRAD_DBIAS_SIDE", "1" if side == "beside" else "0")
    N, Cin, D, H, W, Cout, k, stride, pad, tpad, dt = case
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=450 + Cout, dt=dt,
                                 stride=stride)
    dw, db = c3.conv3d_bwd_weight(x, dy, k, stride, pad, tpad)
    assert c3.poll_status() == c3.Status.OK
    ref_db = oracle.decode16(si.bits(dy), od).reshape(-1, Cout).sum(axis=0)
    assert_close(db.double().cpu().numpy(), ref_db, f"dbias {case} {side}")
    _, ref_dw, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, stride,
                                          pad, tpad)
    assert_close(dw.double().cpu().numpy(), ref_dw, f"dw {case} {side}")


@pytest.mark.parametrize("block", ["1", "0"])
@pytest.mark.parametrize("case", [
    # N, Cin, D, H, W, Cout, kernel, stride, pad, tpad, dtype
    (1, 256, 2, 16, 16, 320, (1, 1, 1), (1, 1, 1), (0, 0, 0), ZERO, "bf16"),   # 2 output tiles, 64 live
    (2, 128, 3, 9, 11, 64, (1, 1, 1), (1, 1, 1), (0, 0, 0), CREP, "f16"),      # ragged frames
    (1, 512, 2, 12, 12, 256, (1, 1, 1), (1, 2, 2), (0, 0, 0), ZERO, "bf16"),   # strided
    (1, 64, 3, 8, 8, 64, (1, 1, 1), (1, 1, 1), (1, 0, 0), ZERO, "bf16"),       # padded end frames
], ids=lambda c: "x".join(map(str, c[:6])) + f"-s{''.join(map(str, c[7]))}-p{c[8][0]}-{c[10]}")
def test_bwd_weight_single_tap_bias_block(case, block, monkeypatch):
    """A single-tap weight gradient sums dy for dbias in one more block of the
    kernel whose A operand is a tile of ones (CONV3D_WGRAD_DBIAS_BLOCK=0: the
    separate pass instead).  With temporal zero padding that leaves output
    frames reading only padding, no tap covers every frame and the separate
    pass runs either way.  dw and dbias against the oracle."""
    monkeypatch.setenv("CONV3D_WGRAD_DBIAS_BLOCK", block)
    N, Cin, D, H, W, Cout, k, stride, pad, tpad, dt = case
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=470 + Cin, dt=dt,
                                 stride=stride)
    dw, db = c3.conv3d_bwd_weight(x, dy, k, stride, pad, tpad)
    assert c3.poll_status() == c3.Status.OK
    ref_db = oracle.decode16(si.bits(dy), od).reshape(-1, Cout).sum(axis=0)
    assert_close(db.double().cpu().numpy(), ref_db, f"dbias {case} block={block}")
    _, ref_dw, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, stride,
                                          pad, tpad)
    assert_close(dw.double().cpu().numpy(), ref_dw, f"dw {case} block={block}")


@pytest.mark.parametrize("mix", ["1", "0"])
@pytest.mark.parametrize("case", [WEIGHT_CASES[i] for i in (0, 2, 6, 7, 11)],
                         ids=lambda c: "x".join(map(str, c[:6])) + f"-p{c[8][0]}-t{c[9]}-{c[10]}")
def test_bwd_weight_swapped_entry_blocks_across_taps(case, mix, monkeypatch):
    """The swapped weight gradient numbers its 64-channel entries across the
    temporal taps (CONV3D_WGRAD_MIX=1, the default where a tap's entries do not
    fill whole blocks): a block may hold entries of two taps, and a tap that
    reads zero padding for a frame loads zeros.  Against the oracle either way,
    including a temporal pad wider than the kernel reaches."""
    monkeypatch.setenv("CONV3D_WGRAD_SWAP", "1")
    monkeypatch.setenv("CONV3D_WGRAD_MIX", mix)
    N, Cin, D, H, W, Cout, k, stride, pad, tpad, dt = case
    if Cin % 64:
        pytest.skip("the swapped weight gradient needs Cin % 64 == 0")
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=490 + Cin, dt=dt,
                                 stride=stride)
    dw, db = c3.conv3d_bwd_weight(x, dy, k, stride, pad, tpad)
    assert c3.poll_status() == c3.Status.OK
    _, ref_dw, ref_db = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, stride,
                                               pad, tpad)
    assert_close(dw.double().cpu().numpy(), ref_dw, f"dw {case} mix={mix}")
    assert_close(db.double().cpu().numpy(), ref_db, f"dbias {case} mix={mix}")


# ------------------------------------------------------ full-size workloads, sampled

from seeded_inputs.workloads import WORKLOADS  # noqa: E402

FULL = ["cfg2", "cfg3", "cfg4s", "cfg5c", "cfg5d", "cfg2s"]


def _full_problem(name):
    wl = WORKLOADS[name]
    x, w, dy, od = grads_problem(wl.N, wl.Cin, wl.D, wl.H, wl.W, wl.Cout, wl.kernel, wl.pad,
                                 wl.tpad, wl.seed, wl.dtype, wl.stride)
    return wl, x, w, dy, od


@pytest.mark.parametrize("name", [n for n in FULL if WORKLOADS[n].stride == (1, 1, 1)])
def test_bwd_data_full_size_sampled(name):
    import numpy as np
    wl, x, w, dy, od = _full_problem(name)
    dx = c3.conv3d_bwd_data(dy, w, x.shape, wl.pad, wl.tpad)
    assert c3.poll_status() == c3.Status.OK
    total = wl.N * wl.D * wl.H * wl.W
    HW = wl.H * wl.W
    rng = np.random.default_rng(5)
    pix = {0, wl.W - 1, HW - 1, HW // 2 + wl.W // 2, total - 1, (wl.D - 1) * HW}
    pix |= {int(v) for v in rng.integers(0, total, 40)}
    pix |= {int(v) for v in rng.integers(0, HW, 16)}    # frame 0: the replicated copies' sum
    pix = np.array(sorted(pix), dtype=np.int64)
    ref = oracle.conv3d_dx_at(si.bits(w), si.bits(dy), od, x.shape, wl.kernel, wl.stride, wl.pad,
                              wl.tpad, pix)
    got = dx.view(-1, wl.Cin)[torch.from_numpy(pix).cuda()].double().cpu().numpy()
    assert_close(got, ref, name)


@pytest.mark.parametrize("name", FULL)
def test_bwd_weight_full_size_sampled(name):
    import numpy as np
    wl, x, w, dy, od = _full_problem(name)
    dw, db = c3.conv3d_bwd_weight(x, dy, wl.kernel, wl.stride, wl.pad, wl.tpad)
    assert c3.poll_status() == c3.Status.OK
    total = dw.numel()
    rng = np.random.default_rng(6)
    ent = {0, total - 1, wl.Cin - 1, total - wl.Cin}
    ent |= {int(v) for v in rng.integers(0, total, 200)}
    ent = np.array(sorted(ent), dtype=np.int64)
    ref = oracle.conv3d_dw_at(si.bits(x), si.bits(dy), od, wl.Cout, wl.kernel, wl.stride, wl.pad,
                              wl.tpad, ent)
    got = dw.view(-1)[torch.from_numpy(ent).cuda()].double().cpu().numpy()
    assert_close(got, ref, name + " dw")
    ref_db = oracle.decode16(si.bits(dy), od).reshape(-1, wl.Cout).sum(axis=0)
    assert_close(db.double().cpu().numpy(), ref_db, name + " dbias")


def test_bwd_data_deterministic_bitwise():
    """dx runs the forward kernel and a fixed-order fold: repeated calls agree bit for bit."""
    x, w, dy, od = grads_problem(2, 64, 4, 10, 12, 64, (3, 3, 3), (0, 1, 1), CREP, 17, "bf16")
    a = c3.conv3d_bwd_data(dy, w, x.shape, (0, 1, 1), CREP)
    b = c3.conv3d_bwd_data(dy, w, x.shape, (0, 1, 1), CREP)
    assert c3.poll_status() == c3.Status.OK
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("combine", ["1", "0"])
@pytest.mark.parametrize("D", [2, 4, 20])
def test_bwd_data_causal_one_launch_on_a_side_stream(D, combine, monkeypatch):
    """Under causal replicate padding one launch computes every frame: with
    CONV3D_DGRAD_COMBINE=1 frame 0's tiles also run the taps of its kt-1
    replicated copies into the same accumulator; with 0 the launch writes the
    kt fp32 parts of frame 0 beside the 16-bit frames 1.. (mixed output) and a
    fold rounds frame 0.  Every element against the oracle, on a stream
    other than the default one, whose later work sees the finished dx."""
    monkeypatch.setenv("CONV3D_DGRAD_COMBINE", combine)
    x, w, dy, od = grads_problem(2, 64, D, 8, 10, 64, (3, 3, 3), (0, 1, 1), CREP, 23, "bf16")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        a = c3.conv3d_bwd_data(dy, w, x.shape, (0, 1, 1), CREP)
        a_copy = a.clone()             # ordered after the call on the same stream
    torch.cuda.synchronize()
    assert c3.poll_status() == c3.Status.OK
    rdx, _, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, (3, 3, 3),
                                       (1, 1, 1), (0, 1, 1), CREP)
    assert_close(a.double().cpu().numpy(), rdx, f"dx D={D}")
    assert torch.equal(a_copy.view(torch.int16), a.view(torch.int16))


@pytest.mark.parametrize("combine", ["1", "0"])
@pytest.mark.parametrize("case", [
    # N, Cin, D, H, W, Cout, kernel, pad, dtype
    (2, 64, 3, 9, 11, 48, (3, 3, 3), (0, 1, 1), "f16"),
    (1, 32, 5, 12, 7, 64, (2, 3, 3), (0, 1, 1), "f16"),      # kt = 2: one replicated copy
    (1, 48, 4, 10, 10, 40, (3, 1, 1), (0, 0, 0), "bf16"),    # temporal taps only
], ids=lambda c: "x".join(map(str, c[:6])) + f"-k{''.join(map(str, c[6]))}-{c[8]}")
def test_bwd_data_causal_front_variants(case, combine, monkeypatch):
    """Both forms of frame 0's gradient under causal replicate padding on fp16,
    kt = 2 and a temporal-only kernel: every element against the oracle."""
    monkeypatch.setenv("CONV3D_DGRAD_COMBINE", combine)
    N, Cin, D, H, W, Cout, k, pad, dt = case
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, CREP, 41 + Cin, dt)
    dx = torch.full(x.shape, float("nan"), dtype=x.dtype, device="cuda")
    dx = c3.conv3d_bwd_data(dy, w, x.shape, pad, CREP, dx=dx)
    assert c3.poll_status() == c3.Status.OK
    ref, _, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, (1, 1, 1), pad,
                                       CREP)
    assert_close(dx.double().cpu().numpy(), ref, f"dx {case} combine={combine}")


@pytest.mark.parametrize("tpad", [CREP, CZERO])
def test_autograd_function_matches_the_oracle(tpad):
    """Conv3dFunction: one backward through the library gives the oracle's adjoints
    for x, w and bias, and dy itself for the residual."""
    N, Cin, D, H, W, Cout, k, pad = 1, 64, 4, 9, 11, 96, (3, 3, 3), (0, 1, 1)
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=31, dt="bf16")
    bias = si.tensor((Cout,), 31, 2, 0.1, torch.bfloat16, "cuda")
    res = si.tensor(dy.shape, 31, 3, 1.0, torch.bfloat16, "cuda")
    leaves = [t.clone().requires_grad_(True) for t in (x, w, bias, res)]
    y = c3.conv3d_autograd(*leaves, pad=pad, tpad=tpad)
    y.backward(dy)
    assert c3.poll_status() == c3.Status.OK
    rdx, rdw, rdb = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, (1, 1, 1),
                                           pad, tpad)
    assert_close(leaves[0].grad.double().cpu().numpy(), rdx, "dx")
    assert_close(leaves[1].grad.double().cpu().numpy(), rdw, "dw")
    assert_close(leaves[2].grad.double().cpu().numpy(), rdb, "dbias")
    assert torch.equal(leaves[3].grad, dy)


STRIDED_DATA_CASES = [
    # N, Cin, D, H, W, Cout, kernel, stride, pad, tpad, dtype
    (1, 64, 3, 16, 16, 64, (3, 3, 3), (1, 2, 2), (0, 1, 1), CREP, "bf16"),   # the downsampling layer
    (2, 64, 3, 15, 17, 128, (3, 3, 3), (1, 2, 2), (0, 1, 1), CZERO, "bf16"), # odd sizes, 2 samples
    (1, 32, 4, 13, 11, 48, (3, 3, 3), (1, 3, 2), (1, 1, 0), ZERO, "f16"),
    (1, 64, 2, 9, 10, 64, (1, 1, 1), (1, 2, 2), (0, 0, 0), ZERO, "bf16"),    # phases without taps
    (1, 64, 1, 12, 12, 64, (3, 3, 3), (1, 2, 2), (0, 1, 1), CREP, "bf16"),   # single frame: fold
    (3, 64, 3, 8, 10, 64, (3, 3, 3), (1, 2, 2), (0, 1, 1), CREP, "bf16"),    # body launch per sample
    (1, 48, 3, 12, 14, 40, (2, 3, 3), (1, 2, 2), (0, 2, 2), CREP, "bf16"),   # pads > kernel - 1
    (1, 64, 2, 10, 9, 64, (3, 3, 3), (1, 1, 2), (0, 1, 1), CZERO, "bf16"),   # one axis strided
]


@pytest.mark.parametrize("case", STRIDED_DATA_CASES, ids=lambda c: "x".join(map(str, c[:6])) + f"-s{''.join(map(str, c[7]))}-t{c[9]}-{c[10]}")
def test_bwd_data_strided_every_element(case, variant):
    N, Cin, D, H, W, Cout, k, stride, pad, tpad, dt = case
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=700 + Cin, dt=dt,
                                 stride=stride)
    dx = torch.full(x.shape, float("nan"), dtype=x.dtype, device="cuda")
    dx = c3.conv3d_bwd_data(dy, w, x.shape, pad, tpad, dx=dx, stride=stride)
    assert c3.poll_status() == c3.Status.OK
    ref, _, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, stride, pad,
                                       tpad)
    assert_close(dx.double().cpu().numpy(), ref, str(case))


@pytest.mark.parametrize("case", [c for c in STRIDED_DATA_CASES if c[9] == CREP and c[2] > 1],
                         ids=lambda c: "x".join(map(str, c[:6])) + f"-s{''.join(map(str, c[7]))}")
def test_bwd_data_strided_combined_front(case, monkeypatch):
    """CONV3D_DGRAD_COMBINE=1 on the strided causal cases (whose few tiles would
    otherwise take the fp32 front frames and the fold): each phase's frame-0
    tiles also run the taps of the replicated copies, straight into dx."""
    monkeypatch.setenv("CONV3D_DGRAD_COMBINE", "1")
    N, Cin, D, H, W, Cout, k, stride, pad, tpad, dt = case
    x, w, dy, od = grads_problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=700 + Cin, dt=dt,
                                 stride=stride)
    dx = torch.full(x.shape, float("nan"), dtype=x.dtype, device="cuda")
    dx = c3.conv3d_bwd_data(dy, w, x.shape, pad, tpad, dx=dx, stride=stride)
    assert c3.poll_status() == c3.Status.OK
    ref, _, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, k, stride, pad,
                                       tpad)
    assert_close(dx.double().cpu().numpy(), ref, str(case))


def test_bwd_data_strided_downsampling_layer_sampled():
    # the 256-channel downsampling workload: 9 frames 256x256 -> 128x128, stride (1, 2, 2)
    from seeded_inputs.workloads import WORKLOADS
    wl = WORKLOADS["cfg2s"]
    x, w, dy, od = grads_problem(wl.N, wl.Cin, wl.D, wl.H, wl.W, wl.Cout, wl.kernel, wl.pad,
                                 wl.tpad, seed=wl.seed, dt=wl.dtype, stride=wl.stride)
    dx = c3.conv3d_bwd_data(dy, w, x.shape, wl.pad, wl.tpad, stride=wl.stride)
    assert c3.poll_status() == c3.Status.OK
    HW = wl.H * wl.W
    pix = sorted({0, 1, wl.W - 1, wl.W, wl.W + 1, HW - 1, HW, 2 * HW + 257, (wl.D - 1) * HW,
                  wl.D * HW - 1} | set(range(5 * HW, 5 * HW + 40)))
    import numpy as np
    pixels = np.array(pix, dtype=np.int64)
    ref = oracle.conv3d_dx_at(si.bits(w), si.bits(dy), od, x.shape, wl.kernel, wl.stride, wl.pad,
                              wl.tpad, pixels)
    got = dx.view(-1, wl.Cin)[torch.from_numpy(pixels).cuda()].double().cpu().numpy()
    assert_close(got, ref, "cfg2s dx sampled")
