"""GPU parity of the decoder-layer neighbours of the GEMV and of the absmean
weight packer, through the C ABI, against the oracle on identical seeded
inputs: int8 codes, x_scale, x_sum, packed bytes and the weight scale
bit-exact; fp32 outputs of the chained FFN block within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_absmax_int8_b200 as tq
from tests._exact import absmean_order_free, rms_order_free
from tests._gpu import assert_y_close, dev, host_pack
from workloads import activations_bf16, make_projections

pytestmark = pytest.mark.gpu
EPS = 1e-5


def f32_of_bf16(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def rms_ref(v, g, eps):
    """The oracle's RMSNorm, after checking that no row's normalising factor
    depends on the order of the fp64 sum of squares: the GPU adds in a tree
    order, the oracle left to right, and the bit-exact comparison below is
    only justified when every order gives the same fp32 factor."""
    assert rms_order_free(v, eps).all(), "an RMSNorm factor depends on the summation order"
    return oracle.rmsnorm(v, g, eps)


def gains(rng, K):
    return rng.uniform(0.5, 1.5, K).astype(np.float32)


def run_rms(M, K, gain, eps, x_bf16=None, x_f32=None, gate=None, up=None):
    xq = torch.full((M, K), -128, dtype=torch.int8, device="cuda")
    xs = torch.full((M,), float("nan"), device="cuda")
    xsum = torch.full((M,), -(2 ** 31), dtype=torch.int32, device="cuda")
    g = dev(gain)
    if gate is not None:
        tq.tq_relu2_mul_rmsnorm_quantize(dev(gate), dev(up), g, eps, xq, xs, xsum, M, K)
    else:
        tq.tq_rmsnorm_quantize(None if x_bf16 is None else dev(x_bf16.view(np.int16)),
                               None if x_f32 is None else dev(x_f32), g, eps, xq, xs, xsum, M, K)
    torch.cuda.synchronize()
    return xq.cpu().numpy(), xs.cpu().numpy(), xsum.cpu().numpy()


def assert_same(got, ref, what):
    q, s, t = got
    rq, rs, rt = ref
    assert np.array_equal(q, rq), f"{what}: codes differ at {np.argwhere(q != rq)[:4].tolist()}"
    assert np.array_equal(s.view(np.uint32), rs.view(np.uint32)), f"{what}: x_scale differs"
    assert np.array_equal(t, rt), f"{what}: x_sum differs"


@pytest.mark.parametrize("M,K", [(1, 2560), (4, 6912), (16, 2560), (3, 16), (2, 32768)])
def test_rmsnorm_quantize_bf16(cuda_device, M, K):
    rng = np.random.default_rng(M * 7 + K)
    xb = activations_bf16(rng, M, K)
    g = gains(rng, K)
    ref = oracle.quant_f32(rms_ref(f32_of_bf16(xb), g, EPS))
    assert_same(run_rms(M, K, g, EPS, x_bf16=xb), ref, f"bf16 M={M} K={K}")


@pytest.mark.parametrize("M,K", [(1, 2560), (5, 6912)])
def test_rmsnorm_quantize_f32(cuda_device, M, K):
    rng = np.random.default_rng(100 + M + K)
    x = (rng.standard_normal((M, K)) * 3).astype(np.float32)
    g = gains(rng, K)
    ref = oracle.quant_f32(rms_ref(x, g, EPS))
    assert_same(run_rms(M, K, g, EPS, x_f32=x), ref, f"f32 M={M} K={K}")


@pytest.mark.parametrize("M,K", [(1, 6912), (8, 6912), (2, 272)])
def test_relu2_mul_rmsnorm_quantize(cuda_device, M, K):
    rng = np.random.default_rng(200 + M + K)
    gate = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    up = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    g = gains(rng, K)
    ref = oracle.quant_f32(rms_ref(oracle.relu2_mul(gate, up), g, EPS))
    assert_same(run_rms(M, K, g, EPS, gate=gate, up=up), ref, f"relu2 M={M} K={K}")


def test_rms_degenerate_rows(cuda_device):
    K = 512
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((4, K)) * 5).astype(np.float32)
    x[1] = 0.0                      # zero row: h = 0, codes 0, scale 0
    x[2] = 2.0                      # constant row, eps = 0: h = gain exactly
    gate = x.copy()
    gate[3] = -1.0                  # relu kills the row: zero codes
    g = gains(rng, K)
    for eps in (0.0, 1.0):
        if eps == 0.0:
            xx = x[[0, 2, 3]]       # eps = 0 with a zero row would divide by 0
            ref = oracle.quant_f32(rms_ref(xx, g, eps))
            assert_same(run_rms(3, K, g, eps, x_f32=xx), ref, "f32 eps=0")
        else:
            ref = oracle.quant_f32(rms_ref(x, g, eps))
            assert_same(run_rms(4, K, g, eps, x_f32=x), ref, "f32 eps=1")
            up = np.ones_like(gate)
            ref = oracle.quant_f32(rms_ref(oracle.relu2_mul(gate, up), g, eps))
            assert_same(run_rms(4, K, g, eps, gate=gate, up=up), ref, "relu2 eps=1")


def y32(acc, w_scale, x_scale):
    """The GEMV epilogue's fp32 rounding order (t = w_scale * x_scale, then
    float(acc) * t), applied to the oracle's exact accumulators."""
    t = np.float32(w_scale) * x_scale.astype(np.float32)
    return acc.astype(np.float32) * t[:, None]


@pytest.mark.parametrize("M,overlap", [(1, False), (4, False), (1, True)])
def test_ffn_block_chain(cuda_device, M, overlap):
    # input RMSNorm + quantiser -> gate, up GEMVs -> relu^2(gate) * up,
    # ffn_sub_norm + quantiser -> down GEMV, each step consuming the last.
    # overlap: the GEMVs as stack launches that stream their weights while
    # the kernel before them runs (the bench's form).
    H, I = 2560, 6912
    gate_p, up_p, down_p = make_projections(
        [("gate_proj", I, H), ("up_proj", I, H), ("down_proj", H, I)], M=M, seed=31 + M)
    rng = np.random.default_rng(77)
    g_in, g_ffn = gains(rng, H), gains(rng, I)
    xb = gate_p.x_bf16                       # the layer input

    # ---- GPU
    P = [dev(host_pack(p.w)) for p in (gate_p, up_p, down_p)]
    xq = torch.empty((M, H), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, device="cuda")
    xsum = torch.empty(M, dtype=torch.int32, device="cuda")
    tq.tq_rmsnorm_quantize(dev(xb.view(np.int16)), None, dev(g_in), EPS, xq, xs, xsum, M, H)
    yg = torch.empty((M, I), device="cuda")
    yu = torch.empty((M, I), device="cuda")
    xq2 = torch.empty((M, I), dtype=torch.int8, device="cuda")
    xs2 = torch.empty(M, device="cuda")
    xsum2 = torch.empty(M, dtype=torch.int32, device="cuda")
    yd = torch.empty((M, H), device="cuda")
    accd = torch.empty((M, H), dtype=torch.int32, device="cuda")
    if overlap:
        ov = tq.TQ_STACK_OVERLAP_PREV
        tq.tq_gemv_stack([tq.make_proj(packed=P[0], xq=xq, x_scale=xs, x_sum=xsum, y=yg,
                                       w_scale=gate_p.w_scale, N=I, K=H),
                          tq.make_proj(packed=P[1], xq=xq, x_scale=xs, x_sum=xsum, y=yu,
                                       w_scale=up_p.w_scale, N=I, K=H)], flags=ov)
        tq.tq_relu2_mul_rmsnorm_quantize(yg, yu, dev(g_ffn), EPS, xq2, xs2, xsum2, M, I)
        tq.tq_gemv_stack([tq.make_proj(packed=P[2], xq=xq2, x_scale=xs2, x_sum=xsum2, y=yd,
                                       acc_out=accd, w_scale=down_p.w_scale, N=H, K=I)],
                         flags=ov)
    else:
        tq.tq_gemv(P[0], gate_p.w_scale, xq, xs, xsum, yg, None, M, I, H)
        tq.tq_gemv(P[1], up_p.w_scale, xq, xs, xsum, yu, None, M, I, H)
        tq.tq_relu2_mul_rmsnorm_quantize(yg, yu, dev(g_ffn), EPS, xq2, xs2, xsum2, M, I)
        tq.tq_gemv(P[2], down_p.w_scale, xq2, xs2, xsum2, yd, accd, M, H, I)
    torch.cuda.synchronize()

    # ---- oracle, the same chain
    q, s, t = oracle.quant_f32(rms_ref(f32_of_bf16(xb), g_in, EPS))
    acc_g = oracle.gemv_threads(oracle.pack(gate_p.w), I, q)
    acc_u = oracle.gemv_threads(oracle.pack(up_p.w), I, q)
    h = oracle.relu2_mul(y32(acc_g, gate_p.w_scale, s), y32(acc_u, up_p.w_scale, s))
    q2, s2, t2 = oracle.quant_f32(rms_ref(h, g_ffn, EPS))
    acc_d = oracle.gemv_threads(oracle.pack(down_p.w), H, q2)
    y_d = oracle.epilogue(acc_d, down_p.w_scale, s2)

    assert_same((xq2.cpu().numpy(), xs2.cpu().numpy(), xsum2.cpu().numpy()), (q2, s2, t2),
                "ffn_sub_norm codes")
    assert np.array_equal(accd.cpu().numpy(), acc_d)
    assert_y_close(yd.cpu().numpy(), y_d)


def run_absmean(Wb):
    N, K = Wb.shape
    packed = torch.full((N // 4, K), 0xFF, dtype=torch.uint8, device="cuda")
    ws = torch.full((1,), float("nan"), device="cuda")
    tq.tq_absmean_pack(dev(Wb.view(np.int16)), packed, ws, N, K)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), ws.cpu().numpy()[0]


@pytest.mark.parametrize("N,K", [(6912, 2560), (2560, 6912), (4, 16), (516, 272)])
def test_absmean_pack_latent_weights(cuda_device, N, K):
    rng = np.random.default_rng(N + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wb = torch.from_numpy(W).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # the fp64 sum of |W| (GPU tree order, oracle left to right) rounds to the
    # same fp32 scale in every order for this input
    assert absmean_order_free(Wb)
    w, g = oracle.absmean(Wb)
    packed, ws = run_absmean(Wb)
    assert np.float32(ws).view(np.uint32) == np.float32(g).view(np.uint32)
    assert np.array_equal(packed, oracle.pack(w))


def test_absmean_pack_dequantised_and_zero(cuda_device):
    # pre-dequantised ternary weights (w * s, exact in bf16) come back as w
    p = next(make_projections([("q_proj", 2560, 2560)], M=1, seed=4))
    Wb = torch.from_numpy(p.w.astype(np.float32) * 0.375).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)
    packed, ws = run_absmean(Wb)
    assert np.array_equal(packed, oracle.pack(p.w))
    assert ws == np.float32(0.375 * np.count_nonzero(p.w) / p.w.size)
    packed, ws = run_absmean(np.zeros((8, 64), np.uint16))
    assert ws == 0 and (packed == 0x55).all()   # every code 1 (weight 0)


@pytest.mark.parametrize("layers", [1, 3])
def test_ffn_block_fused_two_launches(cuda_device, layers):
    # Per layer: one stack launch for gate + up that normalises (RMSNorm,
    # gain g_in) and quantises x itself, then one stack launch for down that
    # computes relu^2(gate) * up, normalises (g_ffn) and quantises -- and
    # streams its weights while the first launch drains. Layers run one
    # after another on the stream.
    H, I = 2560, 6912
    shapes = [(f"L{l}.{n}", a, b) for l in range(layers)
              for (n, a, b) in (("gate_proj", I, H), ("up_proj", I, H), ("down_proj", H, I))]
    projs = list(make_projections(shapes, M=1, seed=90 + layers))
    rng = np.random.default_rng(5)
    gin = [gains(rng, H) for _ in range(layers)]
    gff = [gains(rng, I) for _ in range(layers)]
    keep = []
    out = []
    ov = tq.TQ_STACK_OVERLAP_PREV
    for l in range(layers):
        gp, upp, dp = projs[3 * l:3 * l + 3]
        P = [dev(host_pack(p.w)) for p in (gp, upp, dp)]
        x = dev(gp.x_bf16.view(np.int16))
        g1, g2 = dev(gin[l]), dev(gff[l])
        xq = torch.empty(H, dtype=torch.int8, device="cuda")
        xq_b = torch.empty(H, dtype=torch.int8, device="cuda")
        xs = torch.empty(2, device="cuda")
        xsum = torch.empty(2, dtype=torch.int32, device="cuda")
        yg = torch.empty(I, device="cuda")
        yu = torch.empty(I, device="cuda")
        xq2 = torch.empty(I, dtype=torch.int8, device="cuda")
        xs2 = torch.empty(1, device="cuda")
        xsum2 = torch.empty(1, dtype=torch.int32, device="cuda")
        yd = torch.empty(H, device="cuda")
        accd = torch.empty(H, dtype=torch.int32, device="cuda")
        keep += [P, x, g1, g2]
        # gate and up each quantise the shared input into their own buffers
        tq.tq_gemv_stack([
            tq.make_proj(packed=P[0], x=x, xq=xq, x_scale=xs[0:1], x_sum=xsum[0:1], y=yg,
                         w_scale=gp.w_scale, N=I, K=H, gain=g1, eps=EPS),
            tq.make_proj(packed=P[1], x=x, xq=xq_b, x_scale=xs[1:2], x_sum=xsum[1:2], y=yu,
                         w_scale=upp.w_scale, N=I, K=H, gain=g1, eps=EPS)],
            flags=tq.TQ_STACK_RMSNORM | (ov if l else 0))
        tq.tq_gemv_stack([
            tq.make_proj(packed=P[2], x_f32=yg, up=yu, xq=xq2, x_scale=xs2, x_sum=xsum2, y=yd,
                         acc_out=accd, w_scale=dp.w_scale, N=H, K=I, gain=g2, eps=EPS)],
            flags=tq.TQ_STACK_RELU2_MUL | ov)
        out.append((xq, xq_b, xs, xsum, xq2, xs2, xsum2, yd, accd))
    torch.cuda.synchronize()
    assert tq.tq_device_error(reset=True) == 0

    for l in range(layers):
        gp, upp, dp = projs[3 * l:3 * l + 3]
        xq, xq_b, xs, xsum, xq2, xs2, xsum2, yd, accd = out[l]
        q, s, t = oracle.quant_f32(rms_ref(f32_of_bf16(gp.x_bf16), gin[l], EPS))
        for qq, j in ((xq, 0), (xq_b, 1)):
            assert_same((qq.cpu().numpy()[None], xs.cpu().numpy()[j:j + 1],
                         xsum.cpu().numpy()[j:j + 1]), (q, s, t), f"layer {l} input codes")
        acc_g = oracle.gemv_threads(oracle.pack(gp.w), I, q)
        acc_u = oracle.gemv_threads(oracle.pack(upp.w), I, q)
        h = oracle.relu2_mul(y32(acc_g, gp.w_scale, s), y32(acc_u, upp.w_scale, s))
        q2, s2, t2 = oracle.quant_f32(rms_ref(h, gff[l], EPS))
        assert_same((xq2.cpu().numpy()[None], xs2.cpu().numpy(), xsum2.cpu().numpy()),
                    (q2, s2, t2), f"layer {l} down codes")
        acc_d = oracle.gemv_threads(oracle.pack(dp.w), H, q2)
        assert np.array_equal(accd.cpu().numpy(), acc_d[0])
        assert_y_close(yd.cpu().numpy()[None], oracle.epilogue(acc_d, dp.w_scale, s2))
