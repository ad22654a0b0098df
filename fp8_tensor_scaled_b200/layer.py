"""One FP8-AMAX linear layer step on the device: the whole hot path of the method.

Review page "Training and inference of large language models using 8-bit
floating point", section "Proposed method": every weight, activation and
gradient tensor gets its own amax and bias each step; weights and activations
are cast to FP8_E4 (E4M3), gradients to FP8_E5 (E5M2); the matmuls run on the
FP8 operands and their outputs are unscaled by 2^-(biasA + biasB).

``Fp8AmaxLinear`` owns the FP8 buffers and the per-tensor scalars of one
linear [in -> out] at T tokens, so that a step allocates nothing:

    step(x, w, dy)  ->  quantize X (E4M3), W (E4M3), dY (E5M2)
                        Y  = X8 . W8^T        (fwd)
                        dX = dY8 . W8         (dgrad)
                        dW = dY8^T . X8       (wgrad)

Every operation is one call of the C library (see ``__init__``).
"""
import torch

from . import (E4M3, E5M2, fp8_linear_bwd_dgrad, fp8_linear_bwd_wgrad, fp8_linear_fwd,
               fp8_quantize)


class Fp8AmaxLinear:
    def __init__(self, tokens, in_features, out_features, device, out_dtype=torch.bfloat16,
                 margin_x=0, margin_w=0, margin_dy=0, backward=True):
        self.T, self.inf, self.outf = int(tokens), int(in_features), int(out_features)
        self.margins = (int(margin_x), int(margin_w), int(margin_dy))
        self.backward = backward
        dev = torch.device(device)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.x8 = torch.empty((self.T, self.inf), **u8)
        self.w8 = torch.empty((self.outf, self.inf), **u8)
        # one buffer for the 3 amax values and one for the 3 biases (X, W, dY)
        self.amax = torch.zeros(3, dtype=torch.float32, device=dev)
        self.bias = torch.zeros(3, dtype=torch.int32, device=dev)
        self.y = torch.empty((self.T, self.outf), dtype=out_dtype, device=dev)
        if backward:
            self.dy8 = torch.empty((self.T, self.outf), **u8)
            self.dx = torch.empty((self.T, self.inf), dtype=out_dtype, device=dev)
            self.dw = torch.empty((self.outf, self.inf), dtype=out_dtype, device=dev)

    def quantize(self, x, w, dy=None):
        mx, mw, mdy = self.margins
        fp8_quantize(x, E4M3, mx, self.amax[0:1], self.bias[0:1], self.x8)
        fp8_quantize(w, E4M3, mw, self.amax[1:2], self.bias[1:2], self.w8)
        if self.backward:
            fp8_quantize(dy, E5M2, mdy, self.amax[2:3], self.bias[2:3], self.dy8)

    def gemms(self):
        bx, bw, bdy = self.bias[0:1], self.bias[1:2], self.bias[2:3]
        fp8_linear_fwd(self.x8, E4M3, bx, self.w8, E4M3, bw, out=self.y)
        if self.backward:
            fp8_linear_bwd_dgrad(self.dy8, E5M2, bdy, self.w8, E4M3, bw, out=self.dx)
            fp8_linear_bwd_wgrad(self.dy8, E5M2, bdy, self.x8, E4M3, bx, out=self.dw)

    def step(self, x, w, dy=None):
        self.quantize(x, w, dy)
        self.gemms()
        return (self.y, self.dx, self.dw) if self.backward else (self.y,)

    def flops(self):
        return 2 * self.T * self.inf * self.outf * (3 if self.backward else 1)
