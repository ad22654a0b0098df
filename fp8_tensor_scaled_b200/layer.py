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

    # tensor indices (amax / bias slots) and pass indices
    X, W, DY = 0, 1, 2
    FWD, DGRAD, WGRAD = 0, 1, 2
    # the quantized tensors each pass reads
    PASS_INPUTS = {FWD: (X, W), DGRAD: (DY, W), WGRAD: (DY, X)}

    def begin_step(self):
        """Start a step: returns whether it recomputes amax and bias (refresh)
        or casts with the stored biases."""
        refresh = self.fixed is None and self.calls % self.every == 0
        self.calls += 1
        return refresh

    def quantize_one(self, i, t, refresh):
        """Cast tensor i (X or W to E4M3, dY to E5M2) on the current stream.
        On refresh steps amax -> bias -> cast (fp8_quantize); otherwise cast
        with the stored bias."""
        fmt = E5M2 if i == self.DY else E4M3
        out = (self.x8, self.w8, self.dy8)[i]
        if refresh:
            fp8_quantize(t, fmt, self.margins[i], self.amax[i:i + 1], self.bias[i:i + 1], out)
        else:
            fp8_cast_scaled(t, self.bias[i:i + 1], fmt, out=out)

    def quantize(self, x, w, dy=None):
        """Cast X, W (E4M3) and dY (E5M2)."""
        refresh = self.begin_step()
        self.quantize_one(self.X, x, refresh)
        self.quantize_one(self.W, w, refresh)
        if self.backward:
            self.quantize_one(self.DY, dy, refresh)

    def gemm(self, k):
        """One pass on the current stream: FWD (Y), DGRAD (dX) or WGRAD (dW)."""
        bx, bw, bdy = self.bias[0:1], self.bias[1:2], self.bias[2:3]
        if k == self.FWD:
            fp8_linear_fwd(self.x8, E4M3, bx, self.w8, E4M3, bw, out=self.y)
        elif k == self.DGRAD:
            fp8_linear_bwd_dgrad(self.dy8, E5M2, bdy, self.w8, E4M3, bw, out=self.dx)
        elif self.wgrad_ws is not None:
            fp8_linear_bwd_wgrad_ws(self.dy8, E5M2, bdy, self.x8, E4M3, bx, out=self.dw,
                                    workspace=self.wgrad_ws)
        else:
            fp8_linear_bwd_wgrad(self.dy8, E5M2, bdy, self.x8, E4M3, bx, out=self.dw)

    def outputs(self):
        return (self.y, self.dx, self.dw) if self.backward else (self.y,)

    def gemms(self, pass_done=None):
        """The passes on the current stream.  `pass_done` (optional): one
        CUDA event per pass (fwd, dgrad, wgrad), each recorded as soon as that
        pass's output is complete, so a consumer can take Y before dX and dW
        are done."""
        for k in ((self.FWD, self.DGRAD, self.WGRAD) if self.backward else (self.FWD,)):
            self.gemm(k)
            if pass_done is not None:
                pass_done[k].record()

    def step(self, x, w, dy=None):
        self.quantize(x, w, dy)
        self.gemms()
        return self.outputs()

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
        copies in on one copy stream and out on another, scheduled per tensor
        and per pass so that transfers in both directions overlap each other
        and the compute.  Returns when the caller's stream has been ordered
        after the last copy out.
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
        self.g_done = [torch.cuda.Event() for _ in range(n)]
        self.p_done = [[torch.cuda.Event() for _ in range(3)] for _ in range(n)]
        self.t_in = [[torch.cuda.Event() for _ in range(3)] for _ in range(n)]
        self.t_q = [[torch.cuda.Event() for _ in range(3)] for _ in range(n)]
        self.out_done = torch.cuda.Event()

    def flops(self):
        return sum(l.flops() for l in self.linears)

    def _quantize(self, i, inputs, after=None, timing=None):
        """Quantize linear i's X, W (and dY) in that order on the quantization
        stream, recording an event after each tensor (t_q[i][t]) so that a
        pass can start as soon as its own two operands are ready."""
        stream = self.side if self.overlap else torch.cuda.current_stream(self.device)
        lin = self.linears[i]
        L = Fp8AmaxLinear
        with torch.cuda.stream(stream):
            if after is not None:
                stream.wait_event(after)
            if timing is not None:
                timing["q"][i][0].record(stream)
            refresh = lin.begin_step()
            for t in ((L.X, L.W, L.DY) if lin.backward else (L.X, L.W)):
                lin.quantize_one(t, inputs[i][t], refresh)
                self.t_q[i][t].record(stream)
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
        L = Fp8AmaxLinear
        for i in range(n):
            if i + 1 < n:
                self._quantize(i + 1, inputs, after=in_events[i + 1] if in_events else None,
                               timing=timing)
            lin = self.linears[i]
            passes = (L.FWD, L.DGRAD, L.WGRAD) if lin.backward else (L.FWD,)
            for j, k in enumerate(passes):
                # each pass waits only for its own operands: the forward of
                # the first linear runs while its dY is still being quantized
                for t in L.PASS_INPUTS[k]:
                    main.wait_event(self.t_q[i][t])
                if j == 0 and timing is not None:
                    timing["g"][i][0].record(main)
                lin.gemm(k)
                self.p_done[i][k].record(main)
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

    def host_plan(self):
        """Schedule of the host-buffer step: [(linear, input arrival order,
        pass order), ...].

        The copy out of a pass's output can start only once both of its inputs
        are in, so the copies out trail the copies in at the start of the step
        (the head) and outlast them at the end (the tail: the outputs that
        depend on the last input to arrive).  Per linear the input whose
        dependent outputs are the fewest bytes arrives last, and the pass that
        does not need it runs first; the linear whose first pass needs the
        fewest input bytes goes first, the one with the smallest tail last."""
        L = Fp8AmaxLinear
        plans = []
        for i, l in enumerate(self.linears):
            if not l.backward:
                plans.append((i, (L.W, L.X), (L.FWD,), l.T * l.inf + l.outf * l.inf, 0))
                continue
            ins = {L.X: l.T * l.inf, L.W: l.outf * l.inf, L.DY: l.T * l.outf}
            outs = {L.FWD: l.T * l.outf, L.DGRAD: l.T * l.inf, L.WGRAD: l.outf * l.inf}
            deps = {t: [k for k in outs if t in L.PASS_INPUTS[k]] for t in ins}
            last = min(ins, key=lambda t: (sum(outs[k] for k in deps[t]), t))
            first_pass = next(k for k in outs if last not in L.PASS_INPUTS[k])
            arrival = tuple(t for t in L.PASS_INPUTS[first_pass]) + (last,)
            passes = (first_pass,) + tuple(k for k in (L.FWD, L.DGRAD, L.WGRAD) if k != first_pass)
            head = sum(ins[t] for t in L.PASS_INPUTS[first_pass])
            tail = sum(outs[k] for k in deps[last])
            plans.append((i, arrival, passes, head, tail))
        first = min(plans, key=lambda q: (q[3], q[0]))
        rest = [q for q in plans if q is not first]
        if rest:
            last = min(rest, key=lambda q: (q[4], -q[0]))
            rest = [q for q in rest if q is not last] + [last]
        return [(q[0], q[1], q[2]) for q in [first] + rest]

    def step_from_host(self, host_inputs, device_inputs, host_outputs):
        """One step from pinned host tensors host_inputs[i] = (x, w, dy) into
        the device buffers device_inputs[i], results copied to host_outputs[i]
        = (y, dx, dw).  The copies in run on one stream in the order of
        host_plan(); each tensor is quantized as soon as it has arrived; each
        pass runs as soon as its two operands are quantized; each output
        leaves on a second copy stream as soon as its pass is done."""
        main = torch.cuda.current_stream(self.device)
        qs = self.side if self.overlap else main
        start = torch.cuda.Event()
        start.record(main)
        self.h2d.wait_event(start)          # device inputs free: the previous step is done
        plans = [(i, self.linears[i], arrival, passes) for i, arrival, passes in self.host_plan()]
        L = Fp8AmaxLinear
        with torch.cuda.stream(self.h2d):
            for i, lin, tensors, _ in plans:
                for t in tensors:
                    device_inputs[i][t].copy_(host_inputs[i][t], non_blocking=True)
                    self.t_in[i][t].record(self.h2d)
        for i, lin, tensors, passes in plans:
            refresh = lin.begin_step()
            with torch.cuda.stream(qs):
                for t in tensors:
                    qs.wait_event(self.t_in[i][t])
                    lin.quantize_one(t, device_inputs[i][t], refresh)
                    self.t_q[i][t].record(qs)
            for k in passes:
                for t in L.PASS_INPUTS[k]:
                    main.wait_event(self.t_q[i][t])
                lin.gemm(k)
                self.p_done[i][k].record(main)
        with torch.cuda.stream(self.d2h):
            for i, lin, _, passes in plans:
                outs = lin.outputs()
                for k in passes:
                    self.d2h.wait_event(self.p_done[i][k])
                    host_outputs[i][k].copy_(outs[k], non_blocking=True)
            self.out_done.record(self.d2h)
        main.wait_event(self.out_done)
