"""GPU parity of the FP8 linear passes (fwd, dgrad, wgrad) through the C ABI,
against the oracle's fp64 matmul of the dequantised FP8 codes.

Tolerance (per element): |gpu - ref| <= 1e-3 * sum|a*b| * 2^-(bA+bB) + 1 BF16 ulp
(see tests/parity.py).  Small shapes are compared in full — ragged in every
dimension against the 128 x 256 x 128 tiles — and the layer shapes of the
GPT-111M, Llama-2-7B and Llama-2-70B workloads are compared on sampled
elements and whole 128-row blocks, in the same launch configuration the
benchmark times."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_gemm_close, codes_equal_nan_aware, to_f64, u8

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("fp8_tensor_scaled_b200")
DEV = "cuda"
E4, E5 = fp8.E4M3, fp8.E5M2


def _quant(x_cpu, fmt, margin):
    """Device quantize + the oracle's own quantize of the same bytes."""
    a, b, q = fp8.fp8_quantize(x_cpu.to(DEV), fmt, margin)
    m_ref, b_ref, q_ref = oracle.quantize(x_cpu, fmt, margin)
    assert int(b.item()) == b_ref
    assert codes_equal_nan_aware(u8(q), q_ref.reshape(x_cpu.shape), fmt)
    return q, b, q_ref.reshape(tuple(x_cpu.shape)), b_ref


def _passes(x, w, dy, margins=(0, 0, 0), fx=E4, fw=E4, fdy=E5):
    """Quantize and return everything the passes need (device and oracle sides)."""
    qx, bx, rqx, rbx = _quant(x, fx, margins[0])
    qw, bw, rqw, rbw = _quant(w, fw, margins[1])
    out = dict(x=(qx, bx, rqx, rbx, fx), w=(qw, bw, rqw, rbw, fw))
    if dy is not None:
        out["dy"] = _quant(dy, fdy, margins[2]) + (fdy,)
    return out


def _run(pass_, Q, out_dtype):
    qx, bx, _, _, fx = Q["x"]
    qw, bw, _, _, fw = Q["w"]
    if pass_ == oracle.FWD:
        return fp8.fp8_linear_fwd(qx, fx, bx, qw, fw, bw, out_dtype=out_dtype)
    qdy, bdy, _, _, fdy = Q["dy"]
    if pass_ == oracle.DGRAD:
        return fp8.fp8_linear_bwd_dgrad(qdy, fdy, bdy, qw, fw, bw, out_dtype=out_dtype)
    return fp8.fp8_linear_bwd_wgrad(qdy, fdy, bdy, qx, fx, bx, out_dtype=out_dtype)


def _oracle_args(pass_, Q):
    _, _, rqx, rbx, fx = Q["x"]
    _, _, rqw, rbw, fw = Q["w"]
    if pass_ == oracle.FWD:
        return rqx, fx, rbx, rqw, fw, rbw
    _, _, rqdy, rbdy, fdy = Q["dy"]
    if pass_ == oracle.DGRAD:
        return rqdy, fdy, rbdy, rqw, fw, rbw
    return rqdy, fdy, rbdy, rqx, fx, rbx


def _compare_full(pass_, Q, T, In, Out, out_dtype, what):
    y = _run(pass_, Q, out_dtype)
    torch.cuda.synchronize()
    ref, absref = oracle.linear(pass_, *_oracle_args(pass_, Q), T, In, Out)
    return assert_gemm_close(to_f64(y), ref, absref, what)


def _compare_sampled(pass_, Q, T, In, Out, out_dtype, what, n_samples=1 << 14, block_cols=2048):
    y = _run(pass_, Q, out_dtype)
    torch.cuda.synchronize()
    R, C = y.shape
    rng = np.random.default_rng(1000 + pass_ + R + C)
    rows = rng.integers(0, R, n_samples)
    cols = rng.integers(0, C, n_samples)
    # corners and the last row / column (ragged tile edges)
    rows = np.concatenate([rows, [0, R - 1, R - 1, 0]])
    cols = np.concatenate([cols, [0, C - 1, 0, C - 1]])
    # one whole 128-row block, first `block_cols` columns
    rb = int(rng.integers(0, max(1, R // 128))) * 128
    br, bc = np.meshgrid(np.arange(rb, min(rb + 128, R)), np.arange(min(block_cols, C)),
                         indexing="ij")
    rows = np.concatenate([rows, br.ravel()])
    cols = np.concatenate([cols, bc.ravel()])
    ref, absref = oracle.linear_entries(pass_, *_oracle_args(pass_, Q), T, In, Out, rows, cols)
    got = to_f64(y)[rows, cols]
    return assert_gemm_close(got, ref, absref, what)


def _inputs(T, In, Out, seed, x_scale=1.0, w_scale=0.02, dy_scale=1e-4):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(T, In, generator=g) * x_scale).to(torch.bfloat16)
    w = (torch.randn(Out, In, generator=g) * w_scale).to(torch.bfloat16)
    dy = (torch.randn(T, Out, generator=g) * dy_scale).to(torch.bfloat16)
    return x, w, dy


SMALL = [(1, 16, 16), (77, 48, 80), (128, 128, 256), (200, 272, 400), (333, 256, 528),
         (130, 1040, 144), (257, 384, 768)]


@pytest.mark.parametrize("T,In,Out", SMALL)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_small_shapes_all_passes(T, In, Out, out_dtype):
    x, w, dy = _inputs(T, In, Out, seed=T * 7 + In + Out)
    Q = _passes(x, w, dy)
    for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD):
        _compare_full(p, Q, T, In, Out, out_dtype, "pass %d %s" % (p, (T, In, Out)))


def test_format_mixes_and_margins():
    T, In, Out = 160, 96, 112
    x, w, dy = _inputs(T, In, Out, seed=5)
    for fx, fw, fdy in ((E5, E4, E4), (E4, E5, E5), (E5, E5, E5), (E4, E4, E4)):
        for margins in ((0, 0, 0), (1, 3, 2)):
            Q = _passes(x, w, dy, margins, fx, fw, fdy)
            for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD):
                _compare_full(p, Q, T, In, Out, torch.float32, "mix %s" % ((fx, fw, fdy),))


def test_c0_single_linear_forward_fp32():
    cfg = workloads.C0
    x, w, _ = workloads.linear_inputs(0, 0)
    Q = _passes(x, w, None)
    lin = cfg.linears[0]
    _compare_full(oracle.FWD, Q, cfg.tokens, lin.in_features, lin.out_features, torch.float32, "c0")


def test_empty_tokens():
    In, Out = 64, 32
    z8 = torch.empty((0, In), dtype=torch.uint8, device=DEV)
    dz8 = torch.empty((0, Out), dtype=torch.uint8, device=DEV)
    w8 = torch.zeros((Out, In), dtype=torch.uint8, device=DEV)
    b = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = fp8.fp8_linear_fwd(z8, E4, b, w8, E4, b)
    assert y.shape == (0, Out)
    dx = fp8.fp8_linear_bwd_dgrad(dz8, E5, b, w8, E4, b)
    assert dx.shape == (0, In)
    dw = torch.full((Out, In), 7.0, dtype=torch.bfloat16, device=DEV)
    fp8.fp8_linear_bwd_wgrad(dz8, E5, b, z8, E4, b, out=dw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dw).item() == 0


@pytest.mark.parametrize("li", [0, 1, 2])
def test_c1_gpt111m(li):
    cfg = workloads.C1
    lin = cfg.linears[li]
    x, w, dy = workloads.linear_inputs(1, li)
    Q = _passes(x, w, dy)
    for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD):
        if li == 0:
            _compare_full(p, Q, cfg.tokens, lin.in_features, lin.out_features, torch.bfloat16,
                          "c1 %s pass %d" % (lin.name, p))
        else:
            _compare_sampled(p, Q, cfg.tokens, lin.in_features, lin.out_features, torch.bfloat16,
                             "c1 %s pass %d" % (lin.name, p))


@pytest.mark.parametrize("li", [0, 1, 2])
@pytest.mark.parametrize("margin", [0, 1])
def test_c2_llama7b_mlp(li, margin):
    cfg = workloads.C2
    lin = cfg.linears[li]
    for step in range(2):                      # bias recomputed on re-drawn tensors each step
        x, w, dy = workloads.linear_inputs(2, li, step=step)
        Q = _passes(x, w, dy, (margin, margin, margin))
        for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD):
            _compare_sampled(p, Q, cfg.tokens, lin.in_features, lin.out_features, torch.bfloat16,
                             "c2 %s m%d s%d pass %d" % (lin.name, margin, step, p),
                             n_samples=1 << 12, block_cols=512)


@pytest.mark.parametrize("li", [0, 1, 2, 3])
def test_c3_llama70b(li):
    cfg = workloads.C3
    lin = cfg.linears[li]
    x, w, dy = workloads.linear_inputs(3, li)
    Q = _passes(x, w, dy)
    for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD):
        _compare_sampled(p, Q, cfg.tokens, lin.in_features, lin.out_features, torch.bfloat16,
                         "c3 %s pass %d" % (lin.name, p), n_samples=1 << 12, block_cols=256)


def test_layer_step_matches_oracle():
    """The whole step object (quantize X, W, dY; fwd, dgrad, wgrad) on c1's first linear."""
    cfg = workloads.C1
    lin = cfg.linears[0]
    x, w, dy = workloads.linear_inputs(1, 0, step=3)
    layer = fp8.Fp8AmaxLinear(cfg.tokens, lin.in_features, lin.out_features, DEV)
    y, dx, dw = layer.step(x.to(DEV), w.to(DEV), dy.to(DEV))
    torch.cuda.synchronize()
    _, bx, qx = oracle.quantize(x, E4, 0)
    _, bw, qw = oracle.quantize(w, E4, 0)
    _, bdy, qdy = oracle.quantize(dy, E5, 0)
    T, In, Out = cfg.tokens, lin.in_features, lin.out_features
    qx, qw, qdy = qx.reshape(T, In), qw.reshape(Out, In), qdy.reshape(T, Out)
    for got, (p, A, fa, ba, B, fb, bb) in zip(
            (y, dx, dw), ((oracle.FWD, qx, E4, bx, qw, E4, bw), (oracle.DGRAD, qdy, E5, bdy, qw, E4, bw),
                          (oracle.WGRAD, qdy, E5, bdy, qx, E4, bx))):
        ref, absref = oracle.linear(p, A, fa, ba, B, fb, bb, T, In, Out)
        assert_gemm_close(to_f64(got), ref, absref, "layer pass %d" % p)


def test_bounded_wait_selftest_and_error_word():
    assert fp8.fp8_device_error(clear=False) == (0, 0)      # nothing timed out so far
    assert fp8.fp8_selftest_bounded_wait(50_000_000) == 5   # FP8_ERR_TIMEOUT, then cleared
    assert fp8.fp8_device_error(clear=False) == (0, 0)
    # the context is still usable afterwards
    x = torch.ones(1024, device=DEV)
    assert fp8.fp8_amax(x).item() == 1.0


@pytest.mark.parametrize("T,In,Out", [(200, 272, 400), (128, 256, 256), (333, 256, 528), (1, 16, 16)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fused_output_amax(T, In, Out, out_dtype):
    """fwd / dgrad with the output amax taken in the epilogue: the output is
    bit-identical to the plain call and the amax is exactly max |stored value|
    (checked against the oracle's amax of the GPU output and fp8_amax)."""
    x, w, dy = _inputs(T, In, Out, seed=11 + T)
    Q = _passes(x, w, dy)
    qx, bx, _, _, fx = Q["x"]
    qw, bw, _, _, fw = Q["w"]
    qdy, bdy, _, _, fdy = Q["dy"]
    y, ya = fp8.fp8_linear_fwd(qx, fx, bx, qw, fw, bw, out_dtype=out_dtype, amax=True)
    y0 = fp8.fp8_linear_fwd(qx, fx, bx, qw, fw, bw, out_dtype=out_dtype)
    dx, dxa = fp8.fp8_linear_bwd_dgrad(qdy, fdy, bdy, qw, fw, bw, out_dtype=out_dtype, amax=True)
    dx0 = fp8.fp8_linear_bwd_dgrad(qdy, fdy, bdy, qw, fw, bw, out_dtype=out_dtype)
    torch.cuda.synchronize()
    for got, plain, a in ((y, y0, ya), (dx, dx0, dxa)):
        assert torch.equal(got.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32),
                           plain.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32))
        ref = oracle.amax(got.cpu())
        assert np.float32(a.item()) == ref
        assert fp8.fp8_amax(got).item() == a.item()
    # both passes also against the oracle's GEMM
    _compare_full(oracle.FWD, Q, T, In, Out, out_dtype, "fwd+amax")


def test_fused_output_amax_empty_and_c3():
    b = torch.zeros(1, dtype=torch.int32, device=DEV)
    z8 = torch.empty((0, 64), dtype=torch.uint8, device=DEV)
    w8 = torch.zeros((32, 64), dtype=torch.uint8, device=DEV)
    a = torch.full((1,), 5.0, device=DEV)
    y, ya = fp8.fp8_linear_fwd(z8, E4, b, w8, E4, b, amax=a)
    torch.cuda.synchronize()
    assert ya.item() == 0.0
    # the Llama-2-70B gate projection, fwd and dgrad
    cfg = workloads.C3
    x, w, dy = workloads.linear_inputs(3, 1)
    Q = _passes(x, w, dy)
    qx, bx, _, _, fx = Q["x"]
    qw, bw, _, _, fw = Q["w"]
    qdy, bdy, _, _, fdy = Q["dy"]
    y, ya = fp8.fp8_linear_fwd(qx, fx, bx, qw, fw, bw, amax=True)
    dx, dxa = fp8.fp8_linear_bwd_dgrad(qdy, fdy, bdy, qw, fw, bw, amax=True)
    torch.cuda.synchronize()
    assert fp8.fp8_amax(y).item() == ya.item()
    assert fp8.fp8_amax(dx).item() == dxa.item()
    assert np.float32(ya.item()) == oracle.amax(y.cpu())


def test_bias_update_every_k_and_fixed_bias():
    """Bias recomputed every k-th step only (the page's update-frequency
    question), and FP8-CSCALE fixed biases: the codes the layer casts are the
    oracle's cast with the bias that should be in force at that step."""
    T, In, Out = 96, 128, 160
    layer = fp8.Fp8AmaxLinear(T, In, Out, DEV, bias_update_every=3)
    fixed = fp8.Fp8AmaxLinear(T, In, Out, DEV, fixed_bias=(2, 9, 20))
    held = None
    for step in range(5):
        scale = 4.0 ** step                    # amax changes every step
        x, w, dy = _inputs(T, In, Out, seed=300 + step, x_scale=scale)
        layer.step(x.to(DEV), w.to(DEV), dy.to(DEV))
        fixed.step(x.to(DEV), w.to(DEV), dy.to(DEV))
        torch.cuda.synchronize()
        if step % 3 == 0:
            held = [oracle.quantize(t, f, 0)[1] for t, f in ((x, E4), (w, E4), (dy, E5))]
        assert layer.bias.cpu().tolist() == held, step
        for t, f, i, buf in ((x, E4, 0, layer.x8), (w, E4, 1, layer.w8), (dy, E5, 2, layer.dy8)):
            ref = oracle.cast_scaled(t, held[i], f).reshape(tuple(t.shape))
            assert codes_equal_nan_aware(u8(buf), ref, f), (step, i)
        for t, f, i, buf in ((x, E4, 0, fixed.x8), (w, E4, 1, fixed.w8), (dy, E5, 2, fixed.dy8)):
            ref = oracle.cast_scaled(t, (2, 9, 20)[i], f).reshape(tuple(t.shape))
            assert codes_equal_nan_aware(u8(buf), ref, f), (step, i)
        assert fixed.bias.cpu().tolist() == [2, 9, 20]
        # and the GEMM on those codes is the oracle's
        ref, absref = oracle.linear(oracle.FWD, u8(layer.x8), E4, held[0], u8(layer.w8), E4,
                                    held[1], T, In, Out)
        assert_gemm_close(to_f64(layer.y), ref, absref, "every-3 fwd step %d" % step)


@pytest.mark.parametrize("T", [1, 16, 33, 64, 77, 128, 129])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_split_k_few_tokens(T, out_dtype):
    """Few-token forward with the split-K workspace: full oracle comparison on
    a shape whose K splits, deterministic across calls.  Up to 128 rows the
    ranges run on 128 x 256 tiles; T = 129 takes CTA-pair tiles, split too."""
    In, Out = 12288, 512                     # 2 tiles of 128 x 256, 96 k-blocks
    x, w, _ = _inputs(T, In, Out, seed=500 + T)
    Q = _passes(x, w, None)
    qx, bx, rqx, rbx, fx = Q["x"]
    qw, bw, rqw, rbw, fw = Q["w"]
    assert fp8.fp8_linear_fwd_workspace_size(T, In, Out) > 0
    plan = fp8.fp8_linear_plan(fp8.FWD, T, In, Out, with_workspace=True)
    assert plan["k_splits"] > 1 and plan["tile_m"] == (128 if T <= 128 else 256), plan
    y1 = fp8.fp8_linear_fwd_ws(qx, fx, bx, qw, fw, bw, out_dtype=out_dtype)
    y2 = fp8.fp8_linear_fwd_ws(qx, fx, bx, qw, fw, bw, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    ref, absref = oracle.linear(oracle.FWD, rqx, fx, rbx, rqw, fw, rbw, T, In, Out)
    assert_gemm_close(to_f64(y1), ref, absref, "split-K T=%d" % T)


@pytest.mark.parametrize("li", [3])
def test_split_k_decode_llama70b(li):
    """Decode-sized T on the Llama-2-70B down projection (the one that
    splits: 32 wide tiles, K = 28672), sampled against the oracle."""
    cfg = workloads.C3
    lin = cfg.linears[li]
    T = 16
    x, w, _ = workloads.linear_inputs(3, li)
    x = x[:T].contiguous()
    Q = _passes(x, w, None)
    qx, bx, rqx, rbx, fx = Q["x"]
    qw, bw, rqw, rbw, fw = Q["w"]
    assert fp8.fp8_linear_fwd_workspace_size(T, lin.in_features, lin.out_features) > 0
    y = fp8.fp8_linear_fwd_ws(qx, fx, bx, qw, fw, bw)
    torch.cuda.synchronize()
    rng = np.random.default_rng(li)
    rows = np.repeat(np.arange(T), 64)
    cols = rng.integers(0, lin.out_features, rows.size)
    ref, absref = oracle.linear_entries(oracle.FWD, rqx, fx, rbx, rqw, fw, rbw, T,
                                        lin.in_features, lin.out_features, rows, cols)
    assert_gemm_close(to_f64(y)[rows, cols], ref, absref, "decode %s" % lin.name)


def test_step_from_host_matches_device_step():
    """The host-buffer step (copies in and out scheduled per tensor and per
    pass, linears reordered) gives the device-resident step's results bit for
    bit, and the biases of every linear."""
    from fp8_tensor_scaled_b200.layer import Fp8AmaxStep
    shapes = [(256, 384, 512), (256, 128, 256), (256, 512, 384)]
    dev_l, host_l, inputs = [], [], []
    for i, (T, In, Out) in enumerate(shapes):
        x, w, dy = _inputs(T, In, Out, seed=70 + i)
        inputs.append((x, w, dy))
        dev_l.append(fp8.Fp8AmaxLinear(T, In, Out, DEV))
        host_l.append(fp8.Fp8AmaxLinear(T, In, Out, DEV))
    d_in = [tuple(t.to(DEV) for t in inp) for inp in inputs]
    scratch = [tuple(torch.empty_like(t) for t in inp) for inp in d_in]
    h_in = [tuple(t.pin_memory() for t in inp) for inp in inputs]
    h_out = [tuple(torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in l.outputs())
             for l in host_l]
    a, b = Fp8AmaxStep(dev_l), Fp8AmaxStep(host_l)
    for _ in range(2):
        a.step(d_in)
        b.step_from_host(h_in, scratch, h_out)
    torch.cuda.synchronize()
    for la, lb, ho in zip(dev_l, host_l, h_out):
        assert torch.equal(la.bias, lb.bias)
        for o, h in zip(la.outputs(), ho):
            assert torch.equal(o.cpu(), h)


def test_plan_query_errors():
    with pytest.raises(fp8.Fp8Error) as e:
        fp8.fp8_linear_plan(7, 16, 16, 16)
    assert e.value.status == 1
    with pytest.raises(fp8.Fp8Error):
        fp8.fp8_linear_plan(fp8.FWD, -1, 16, 16)
    # decode-sized forward without a workspace: narrow 128 x 64 tiles
    assert fp8.fp8_linear_plan(fp8.FWD, 16, 8192, 8192)["tile_n"] == 64


def test_split_k_workspace_errors():
    T, In, Out = 8, 12288, 512
    x8 = torch.zeros((T, In), dtype=torch.uint8, device=DEV)
    w8 = torch.zeros((Out, In), dtype=torch.uint8, device=DEV)
    b = torch.zeros(1, dtype=torch.int32, device=DEV)
    small = torch.empty(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(fp8.Fp8Error) as e:
        fp8.fp8_linear_fwd_ws(x8, E4, b, w8, E4, b, workspace=small)
    assert e.value.status == 1
    # a problem that does not split needs no workspace
    assert fp8.fp8_linear_fwd_workspace_size(4096, 1024, 4096) == 0


def test_step_graph_replay_matches_eager():
    """A multi-linear step recorded into a CUDA graph replays the same
    kernels: outputs, biases and codes equal the eager step's bit for bit."""
    from fp8_tensor_scaled_b200.layer import Fp8AmaxStep
    shapes = [(256, 384, 512), (256, 512, 256)]
    inputs, eager_l, graph_l = [], [], []
    for i, (T, In, Out) in enumerate(shapes):
        x, w, dy = _inputs(T, In, Out, seed=900 + i)
        inputs.append((x.to(DEV), w.to(DEV), dy.to(DEV)))
        eager_l.append(fp8.Fp8AmaxLinear(T, In, Out, DEV))
        graph_l.append(fp8.Fp8AmaxLinear(T, In, Out, DEV))
    eager = Fp8AmaxStep(eager_l)
    graph = Fp8AmaxStep(graph_l)
    graph.capture(inputs)
    for _ in range(2):
        eager.step(inputs)
        graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager_l, graph_l):
        for name in ("y", "dx", "dw", "x8", "w8", "dy8", "bias", "amax"):
            assert torch.equal(getattr(a, name), getattr(b, name)), name
    with pytest.raises(ValueError):
        Fp8AmaxStep([fp8.Fp8AmaxLinear(16, 16, 16, DEV, bias_update_every=2)]).capture(
            [(inputs[0][0][:16, :16].contiguous(), inputs[0][1][:16, :16].contiguous(),
              inputs[0][2][:16, :16].contiguous())])


@pytest.mark.parametrize("T,In,Out", [(8192, 768, 768), (4096, 512, 256), (3000, 256, 640)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_split_k_small_weight_gradient(T, In, Out, out_dtype):
    """Small dW over many tokens: CTA-pair tiles split along K (T) through the
    workspace entry point, full oracle comparison, deterministic."""
    assert fp8.fp8_linear_bwd_wgrad_workspace_size(T, In, Out) > 0
    plan = fp8.fp8_linear_plan(fp8.WGRAD, T, In, Out, with_workspace=True)
    assert plan["ctas_per_tile"] == 2 and plan["k_splits"] > 1, plan
    assert fp8.fp8_linear_plan(fp8.WGRAD, T, In, Out)["k_splits"] == 1
    x, w, dy = _inputs(T, In, Out, seed=T + In + Out)
    Q = _passes(x, w, dy)
    qx, bx, rqx, rbx, fx = Q["x"]
    qdy, bdy, rqdy, rbdy, fdy = Q["dy"]
    a = fp8.fp8_linear_bwd_wgrad_ws(qdy, fdy, bdy, qx, fx, bx, out_dtype=out_dtype)
    b = fp8.fp8_linear_bwd_wgrad_ws(qdy, fdy, bdy, qx, fx, bx, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    ref, absref = oracle.linear(oracle.WGRAD, rqdy, fdy, rbdy, rqx, fx, rbx, T, In, Out)
    assert_gemm_close(to_f64(a), ref, absref, "split-K wgrad %s" % ((T, In, Out),))


# Problems of many tiles run on 256 x 512 CTA-pair tiles (two M=256, N=256
# MMAs per K step sharing the A stage, one 512-column accumulator drained in
# two halves).  The shapes below are in that regime and ragged in every
# dimension: 9 row blocks (the last one partly filled); N = 8000 leaves 320
# columns in the last 512-column block (64 in its second half), N = 7696
# leaves 16 (its second half empty: neither loaded nor multiplied); K ragged
# against the 128-wide k-blocks.  Every element of rows and columns at the
# tile and half-tile edges is checked, plus random samples.
@pytest.mark.parametrize("N", [8000, 7696])
@pytest.mark.parametrize("pass_", [oracle.FWD, oracle.DGRAD, oracle.WGRAD])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_double_width_tiles(N, pass_, out_dtype):
    if pass_ == oracle.FWD:
        T, In, Out = 2148, 400, N
    elif pass_ == oracle.DGRAD:
        T, In, Out = 2148, N, 400
    else:
        T, In, Out = 300, N, 2160
    plan = fp8.fp8_linear_plan(pass_, T, In, Out)
    assert (plan["tile_m"], plan["tile_n"], plan["ctas_per_tile"], plan["k_splits"]) == \
        (256, 512, 2, 1), plan
    x, w, dy = _inputs(T, In, Out, seed=N + 10 * pass_)
    Q = _passes(x, w, None if pass_ == oracle.FWD else dy)
    y = _run(pass_, Q, out_dtype)
    torch.cuda.synchronize()
    R, C = y.shape
    edge_rows = sorted({0, 1, 127, 128, 255, 256, R - 101, R - 100, R - 1})
    last = (C - 1) // 512 * 512
    edge_cols = sorted({0, 31, 32, 255, 256, 511, 512, last - 1, last, last + 255, last + 256,
                        C - 1} & set(range(C)))
    rng = np.random.default_rng(N + pass_)
    parts_r = [rng.integers(0, R, 1 << 14)]
    parts_c = [rng.integers(0, C, 1 << 14)]
    for r in edge_rows:
        parts_r.append(np.full(C, r))
        parts_c.append(np.arange(C))
    for c in edge_cols:
        parts_r.append(np.arange(R))
        parts_c.append(np.full(R, c))
    rows, cols = np.concatenate(parts_r), np.concatenate(parts_c)
    ref, absref = oracle.linear_entries(pass_, *_oracle_args(pass_, Q), T, In, Out, rows, cols)
    assert_gemm_close(to_f64(y)[rows, cols], ref, absref, "double tile pass %d %s" % (pass_, (T, In, Out)))


def test_concurrent_host_threads():
    """Calls from several host threads at once, each on its own stream (ctypes
    releases the GIL during the call), give the results of serial calls."""
    import threading
    shapes = [(200, 272, 400), (1024, 512, 1024), (16, 4096, 512), (333, 256, 528)]
    cases = []
    for i, (T, In, Out) in enumerate(shapes):
        x, w, dy = _inputs(T, In, Out, seed=900 + i)
        cases.append(_passes(x, w, dy))
    ref = [[_run(p, Q, torch.bfloat16) for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD)]
           for Q in cases]
    torch.cuda.synchronize()
    out = [None] * len(cases)
    errors = []

    def work(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(3):
                    r = [_run(p, cases[i], torch.bfloat16)
                         for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD)]
                s.synchronize()
            out[i] = r
        except Exception as e:          # reported below, in the test's thread
            errors.append(e)

    threads = [threading.Thread(target=work, args=(i,)) for i in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for a, b in zip(ref, out):
        for x, y in zip(a, b):
            assert torch.equal(x, y)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_unscale_exponent_beyond_normal_range(out_dtype):
    """Tiny tensors give biases near 66 (E4M3) and 73 (E5M2), so the GEMM's
    unscale 2^-(bA+bB) has an exponent below -126, outside what one fp32
    power of two holds: the epilogue applies it as split multiplies.  The
    products stay normal numbers, so the results are compared in full."""
    T, In, Out = 200, 272, 400
    x, w, dy = _inputs(T, In, Out, seed=77, x_scale=2.0 ** -60, w_scale=2.0 ** -60,
                       dy_scale=2.0 ** -60)
    Q = _passes(x, w, dy)
    bx, bw, bdy = Q["x"][3], Q["w"][3], Q["dy"][3]
    assert bx + bw > 127 and bdy + bw > 127 and bdy + bx > 127, (bx, bw, bdy)
    for p in (oracle.FWD, oracle.DGRAD, oracle.WGRAD):
        _compare_full(p, Q, T, In, Out, out_dtype, "split unscale pass %d" % p)
