"""One FP8-AMAX linear layer step on the device: the whole hot path of the method.

Review page "Training and inference of large language models using 8-bit
floating point", section "Proposed method": every weight, activation and
gradient tensor gets its own amax and bias each step; weights and activations
are cast to FP8_E4 (E4M3), gradients to FP8_E5 (E5M2); the matmuls run on the
FP8 operands and their outputs are unscaled by 2^-(biasA + biasB).

``Fp8AmaxLinear`` owns the FP8 buffers and the per-tensor scalars of one
linear [in -> out] at T tokens, so that a step allocates nothing.  Two options
follow the page's comparison of scaling policies ("Proposed method" and the
research questions on how often the bias must be updated):
  * ``bias_update_every=k``: amax and bias are recomputed on every k-th
    step only; the steps in between cast with the stored biases and skip the
    amax pass (k = 1 is FP8-AMAX proper);
  * ``fixed_bias=(bx, bw, bdy)``: FP8-CSCALE, constant biases, no amax at all.

    step(x, w, dy)  ->  quantize X (E4M3), W (E4M3), dY (E5M2)
                        Y  = X8 . W8^T        (fwd)
                        dX = dY8 . W8         (dgrad)
                        dW = dY8^T . X8       (wgrad)

Every operation is one call of the C library (see ``__init__``).
"""
import torch

from . import (E4M3, E5M2, fp8_cast_scaled, fp8_linear_bwd_dgrad, fp8_linear_bwd_wgrad,
               fp8_linear_bwd_wgrad_workspace_size, fp8_linear_bwd_wgrad_ws, fp8_linear_fwd,
               fp8_quantize)


class Fp8AmaxLinear:
    def __init__(self, tokens, in_features, out_features, device, out_dtype=torch.bfloat16,
                 margin_x=0, margin_w=0, margin_dy=0, backward=True, bias_update_every=1,
                 fixed_bias=None):
        self.T, self.inf, self.outf = int(tokens), int(in_features), int(out_features)
        self.margins = (int(margin_x), int(margin_w), int(margin_dy))
        self.backward = backward
        if int(bias_update_every) < 1:
            raise ValueError("bias_update_every must be >= 1")
        self.every = int(bias_update_every)
        self.fixed = tuple(int(b) for b in fixed_bias) if fixed_bias is not None else None
        self.calls = 0
        dev = torch.device(device)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.x8 = torch.empty((self.T, self.inf), **u8)
        self.w8 = torch.empty((self.outf, self.inf), **u8)
        # one buffer for the 3 amax values and one for the 3 biases (X, W, dY)
        self.amax = torch.zeros(3, dtype=torch.float32, device=dev)
        self.bias = torch.zeros(3, dtype=torch.int32, device=dev)
        if self.fixed is not None:
            if len(self.fixed) != 3:
                raise ValueError("fixed_bias is (bias_x, bias_w, bias_dy)")
            self.bias.copy_(torch.tensor(self.fixed, dtype=torch.int32))
        self.y = torch.empty((self.T, self.outf), dtype=out_dtype, device=dev)
        self.wgrad_ws = None
        if backward:
            self.dy8 = torch.empty((self.T, self.outf), **u8)
            self.dx = torch.empty((self.T, self.inf), dtype=out_dtype, device=dev)
            self.dw = torch.empty((self.outf, self.inf), dtype=out_dtype, device=dev)
            # a small dW over many tokens splits K across more CTA pairs
            ws = fp8_linear_bwd_wgrad_workspace_size(self.T, self.inf, self.outf)
            if ws > 0:
                self.wgrad_ws = torch.empty(ws, **u8)

    def quantize(self, x, w, dy=None):
        """Cast X, W (E4M3) and dY (E5M2).  On refresh steps amax -> bias ->
        cast (fp8_quantize); otherwise cast with the stored bias."""
        refresh = self.fixed is None and self.calls % self.every == 0
        self.calls += 1
        work = [(x, E4M3, 0, self.x8), (w, E4M3, 1, self.w8)]
        if self.backward:
            work.append((dy, E5M2, 2, self.dy8))
        for t, fmt, i, out in work:
            if refresh:
                fp8_quantize(t, fmt, self.margins[i], self.amax[i:i + 1], self.bias[i:i + 1], out)
            else:
                fp8_cast_scaled(t, self.bias[i:i + 1], fmt, out=out)

    def gemms(self, pass_done=None):
        """The three GEMMs on the current stream.  `pass_done` (optional): one
        CUDA event per pass (fwd, dgrad, wgrad), each recorded as soon as that
        pass's output is complete, so a consumer can take Y before dX and dW
        are done."""
        bx, bw, bdy = self.bias[0:1], self.bias[1:2], self.bias[2:3]
        fp8_linear_fwd(self.x8, E4M3, bx, self.w8, E4M3, bw, out=self.y)
        if pass_done is not None:
            pass_done[0].record()
        if self.backward:
            fp8_linear_bwd_dgrad(self.dy8, E5M2, bdy, self.w8, E4M3, bw, out=self.dx)
            if pass_done is not None:
                pass_done[1].record()
            if self.wgrad_ws is not None:
                fp8_linear_bwd_wgrad_ws(self.dy8, E5M2, bdy, self.x8, E4M3, bx, out=self.dw,
                                        workspace=self.wgrad_ws)
            else:
                fp8_linear_bwd_wgrad(self.dy8, E5M2, bdy, self.x8, E4M3, bx, out=self.dw)
            if pass_done is not None:
                pass_done[2].record()

    def step(self, x, w, dy=None):
        self.quantize(x, w, dy)
        self.gemms()
        return (self.y, self.dx, self.dw) if self.backward else (self.y,)

    def flops(self):
        return 2 * self.T * self.inf * self.outf * (3 if self.backward else 1)


class Fp8AmaxStep:
    """The fwd+bwd step of several FP8-AMAX linears on one device.

    The GEMMs are tensor-core bound and leave most of the HBM bandwidth idle;
    the amax and cast kernels are HBM bound and need no tensor memory and
    little shared memory, so their blocks fit beside a GEMM's one-CTA-per-SM
    grid.  With ``overlap`` the quantization of linear i+1 therefore runs on a
    side stream while the GEMMs of linear i run on the caller's stream (events
    order every consumer after its producer); without it everything runs in
    order on the caller's stream.  (On a B200 at its power cap the two orders
    measure within a few percent of each other: the step is bound by the
    energy of its work rather than by the order of it.)

    ``step(inputs)``            inputs already on the device: [(x, w, dy), ...]
    ``capture(inputs)`` / ``replay()``  the same step recorded once into a CUDA
        graph (on these input and output buffers) and replayed with a single
        host call: no per-kernel launch cost, which matters for small layers.
    ``step_from_host(h_in, d_in, h_out)``  the same step from pinned host tensors:
        copies in on one copy stream, copies of each linear's Y, dX, dW out on
        another as soon as the pass that writes it finishes, so transfers in both directions
        overlap each other and the compute.  Returns when the caller's stream
        has been ordered after the last copy out.
    """

    def __init__(self, linears, overlap=True):
        self.linears = list(linears)
        dev = self.linears[0].x8.device
        self.device = dev
        self.overlap = overlap
        self.side = torch.cuda.Stream(dev) if overlap else None
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        n = len(self.linears)
        self.q_done = [torch.cuda.Event() for _ in range(n)]
        self.in_done = [torch.cuda.Event() for _ in range(n)]
        self.g_done = [torch.cuda.Event() for _ in range(n)]
        self.p_done = [[torch.cuda.Event() for _ in range(3)] for _ in range(n)]
        self.out_done = torch.cuda.Event()

    def flops(self):
        return sum(l.flops() for l in self.linears)

    def _quantize(self, i, inputs, after=None, timing=None):
        stream = self.side if self.overlap else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(stream):
            if after is not None:
                stream.wait_event(after)
            if timing is not None:
                timing["q"][i][0].record(stream)
            self.linears[i].quantize(*inputs[i])
            if timing is not None:
                timing["q"][i][1].record(stream)
            self.q_done[i].record(stream)

    def step(self, inputs, timing=None, in_events=None):
        """`timing` (optional): {"q": [[ev, ev]] * n, "g": [[ev, ev]] * n} CUDA
        events recorded around each linear's quantization and GEMMs."""
        main = torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(main)
        n = len(self.linears)
        # linear 0 is quantized first; every later one while the previous GEMMs run
        self._quantize(0, inputs, after=in_events[0] if in_events else start, timing=timing)
        for i in range(n):
            if i + 1 < n:
                self._quantize(i + 1, inputs, after=in_events[i + 1] if in_events else None,
                               timing=timing)
            main.wait_event(self.q_done[i])
            if timing is not None:
                timing["g"][i][0].record(main)
            self.linears[i].gemms(self.p_done[i])
            if timing is not None:
                timing["g"][i][1].record(main)
            self.g_done[i].record(main)

    def capture(self, inputs):
        """Record one step into a CUDA graph.  The graph replays the exact
        kernels recorded, so the per-step host decisions must be fixed: every
        linear recomputes its biases every step (bias_update_every == 1) or
        uses fixed biases."""
        if any(l.fixed is None and l.every != 1 for l in self.linears):
            raise ValueError("a captured step needs bias_update_every == 1 or fixed biases")
        dev = self.device
        warm = torch.cuda.Stream(dev)
        warm.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(warm):          # first calls set up per-device state
            self.step(inputs)
        torch.cuda.current_stream(dev).wait_stream(warm)
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step(inputs)
        return self.graph

    def replay(self):
        self.graph.replay()

    def step_from_host(self, host_inputs, device_inputs, host_outputs):
        main = torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(main)
        with torch.cuda.stream(self.h2d):
            self.h2d.wait_event(start)       # device inputs free: the previous step is done
            for i, (hs, ds) in enumerate(zip(host_inputs, device_inputs)):
                for h, d in zip(hs, ds):
                    d.copy_(h, non_blocking=True)
                self.in_done[i].record(self.h2d)
        self.step(device_inputs, in_events=self.in_done)
        with torch.cuda.stream(self.d2h):
            # each output leaves as soon as its own pass is done: the copy of
            # Y overlaps dgrad and wgrad, so the last copy out starts earlier
            for i, (lin, hs) in enumerate(zip(self.linears, host_outputs)):
                for k, (h, d) in enumerate(zip(hs, (lin.y, lin.dx, lin.dw))):
                    self.d2h.wait_event(self.p_done[i][k])
                    h.copy_(d, non_blocking=True)
            self.out_done.record(self.d2h)
        main.wait_event(self.out_done)
