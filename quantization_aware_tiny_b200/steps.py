"""Multi-call sequences of the C-ABI entry points: the depth-recurrent core and
the tied-head + MLP training step.  Only sequencing and buffer ownership live
here; every arithmetic step runs in the library's kernels.
"""
import torch

from . import qat


class RecurrentCore:
    """Depth-recurrent core ("Depth Recurrence + Mixed-Precision Quant"
    write-up, "Stem / Core / Tail" and "税 1"): the block's weights are
    quantized ONCE (the cache) and its linears are applied R times.

    Per application, attention left out (the O projection reads the query
    slice of QKV in its place):
        qkv = x Wqkv^T              (Q|K|V fused: per-row quantization is per
                                     output row, so concatenation is exact)
        x1  = x + q Wo^T            (residual fused in the GEMM epilogue)
        x   = x1 + proj(act(fc(x1)))
    act = relu^2, or leaky_relu(., 0.5)^2 with act="leaky2"; bits = 5 selects
    the int5 grid (the write-up's MLP_INT5 / ATTN_INT5 configuration).
    """

    def __init__(self, Wq, Wk, Wv, Wo, Wfc, Wproj, bits=6, stream=None, act="relu2"):
        self.d = Wq.shape[1]
        self.H = Wfc.shape[0]
        self.bits = bits
        self.act = act
        Wqkv = torch.cat([Wq, Wk, Wv], dim=0).contiguous()
        self.W = (Wqkv, Wo.contiguous(), Wfc.contiguous(), Wproj.contiguous())
        self.q_qkv, self.q_o, self.q_fc, self.q_proj = qat.quantize_weights(self.W, bits,
                                                                             stream=stream)
        self.nqkv = Wqkv.shape[0]
        self._buf = None

    def _buffers(self, T, device):
        if self._buf is None or self._buf[0].shape[0] != T:
            bf = torch.bfloat16
            self._buf = (torch.empty((T, self.nqkv), dtype=bf, device=device),
                         torch.empty((T, self.d), dtype=bf, device=device),
                         torch.empty((T, self.H), dtype=bf, device=device))
        return self._buf

    def forward(self, x, R, stream=None, noise=None):
        """Applies the core R times to x [T,d] bf16 in place; returns x.

        noise = (seed, offset) switches to Noisy QAT ("Depth Recurrence +
        Mixed-Precision Quant", "幸存发现 1"): every application draws fresh
        uniform noise at the int8 step (the int5 step when bits = 5) for each
        of the four weights, with
        Philox offsets offset + 4*r + k (r = application, k = qkv, o, fc,
        proj), instead of reusing the once-quantized operands."""
        T = x.shape[0]
        qkv, x1, h = self._buffers(T, x.device)
        ops = (self.q_qkv, self.q_o, self.q_fc, self.q_proj)
        if noise is not None:
            ops = tuple(qat.QWeight(torch.empty_like(q.operand), None, None, 0) for q in ops)
        for r in range(R):
            if noise is not None:
                seed, offset = noise
                for k, (w, q) in enumerate(zip(self.W, ops)):
                    qat.qat_noisy_operand(w, seed, offset + 4 * r + k, q.operand, stream=stream,
                                          bits=self.bits)
            q_qkv, q_o, q_fc, q_proj = ops
            bits = self.bits
            qat.qat_linear_fwd(x, qkv, bits, qw=q_qkv, stream=stream)
            qat.qat_linear_fwd(qkv, x1, bits, qw=q_o, ldx=self.nqkv, T=T, residual=x, stream=stream)
            qat.qat_mlp_fwd(x1, x, bits, self.d, self.H, qfc=q_fc, qproj=q_proj, residual=x1,
                            h_save=h, stream=stream, act=self.act)
        return x

    # ------------------------------------------------------------- training

    def _ops_for_noise(self, noise, R, stream):
        """Noisy QAT operands of every application (kept for the backward):
        application r draws weight k at Philox offset offset + 4*r + k."""
        seed, offset = noise
        apps = []
        for r in range(R):
            ops = tuple(qat.QWeight(torch.empty_like(q.operand), None, None, 0)
                        for q in (self.q_qkv, self.q_o, self.q_fc, self.q_proj))
            for k, (w, q) in enumerate(zip(self.W, ops)):
                qat.qat_noisy_operand(w, seed, offset + 4 * r + k, q.operand, stream=stream,
                                      bits=self.bits)
            apps.append(ops)
        return apps

    def forward_train(self, x, R, stream=None, noise=None):
        """The forward of forward() for training: x [T,d] bf16 is left as it is
        and every application's activations are kept for backward() -- its
        input state, qkv, x1, pre, h and output state.  Returns the output
        state of the last application (a buffer the core owns)."""
        T, dev, bf = x.shape[0], x.device, torch.bfloat16
        e = lambda n: torch.empty((T, n), dtype=bf, device=dev)
        apps = self._ops_for_noise(noise, R, stream) if noise is not None else \
            [(self.q_qkv, self.q_o, self.q_fc, self.q_proj)] * R
        saved = []
        xin = x
        for r in range(R):
            s = {"x": xin, "qkv": e(self.nqkv), "x1": e(self.d), "pre": e(self.H),
                 "h": e(self.H), "out": e(self.d), "ops": apps[r]}
            q_qkv, q_o, q_fc, q_proj = apps[r]
            qat.qat_linear_fwd(xin, s["qkv"], self.bits, qw=q_qkv, stream=stream)
            qat.qat_linear_fwd(s["qkv"], s["x1"], self.bits, qw=q_o, ldx=self.nqkv, T=T,
                               residual=xin, stream=stream)
            qat.qat_mlp_fwd(s["x1"], s["out"], self.bits, self.d, self.H, qfc=q_fc, qproj=q_proj,
                            residual=s["x1"], pre_save=s["pre"], h_save=s["h"], stream=stream,
                            act=self.act)
            saved.append(s)
            xin = s["out"]
        self._saved = saved
        return xin

    def _grad_buffers(self, T, device):
        if getattr(self, "_gbuf", None) is None or self._gbuf["dx1"].shape[0] != T:
            bf, f32 = torch.bfloat16, torch.float32
            e = lambda *sh, dt=bf: torch.empty(sh, dtype=dt, device=device)
            self._gbuf = {"dx1": e(T, self.d), "dq": e(T, self.d), "g": (e(T, self.d), e(T, self.d)),
                          "ws": e(qat.workspace_size(qat.QAT_OP_MLP_BWD, self.d, self.H, T, False),
                                  dt=torch.uint8)}
            self.dWqkv = e(self.nqkv, self.d, dt=f32)
            self.dWo = e(self.d, self.d, dt=f32)
            self.dWfc = e(self.H, self.d, dt=f32)
            self.dWproj = e(self.d, self.H, dt=f32)
        return self._gbuf

    def backward_application(self, s, g, dx, accumulate, stream=None):
        """STE backward of one application from its saved activations s (x,
        qkv, x1, pre, h and its operands) and g = dL/d out; writes dL/dx into
        dx and adds (accumulate) or writes the application's weight gradients
        into dWqkv, dWo, dWfc, dWproj:
            dx1 = g + dpre Wfc      (qat_mlp_bwd, residual fused; dWfc, dWproj)
            dq  = dx1 Wo            (qat_linear_bwd on the query slice of qkv; dWo)
            dx  = dx1 + dq Wq       (qat_linear_bwd, residual fused; dWq)
        K and V do not reach the output with attention left out: their rows of
        dWqkv are zeroed when not accumulating and otherwise left as they are."""
        T = g.shape[0]
        gb = self._grad_buffers(T, g.device)
        q_qkv, q_o, q_fc, q_proj = s["ops"]
        d = self.d
        qat.qat_mlp_bwd(s["x1"], s["pre"], s["h"], g, self.bits, d, self.H, qfc=q_fc,
                        qproj=q_proj, dX=gb["dx1"], dX_residual=g, dWfc=self.dWfc,
                        dWproj=self.dWproj, accumulate_dW=accumulate, workspace=gb["ws"],
                        stream=stream, act=self.act)
        qat.qat_linear_bwd(s["qkv"], gb["dx1"], self.bits, qw=q_o, dX=gb["dq"], dW=self.dWo,
                           accumulate_dW=accumulate, ldx=self.nqkv, stream=stream)
        q_q = qat.QWeight(q_qkv.operand[:d], None, None, self.bits)
        qat.qat_linear_bwd(s["x"], gb["dq"], self.bits, qw=q_q, dX=dx, dX_residual=gb["dx1"],
                           dW=self.dWqkv[:d], accumulate_dW=accumulate, stream=stream)
        if not accumulate:  # T = 0 call: zeroes the k|v rows of dWqkv
            qat.qat_linear_bwd(None, gb["dq"][:0], self.bits, dW=self.dWqkv[d:],
                               N=self.nqkv - d, K=d, stream=stream)

    def backward(self, dY, stream=None, accumulate=False):
        """Backward through the applications of the last forward_train, in
        reverse (P1 "税 1": the shared weights' gradients are summed over the R
        uses).  dY = dL/d(output state) [T,d] bf16.  Returns dL/dx (a buffer
        the core owns); weight gradients in dWqkv, dWo, dWfc, dWproj (fp32,
        overwritten, or added to with accumulate=True)."""
        gb = self._grad_buffers(dY.shape[0], dY.device)
        g = dY
        for i, r in enumerate(reversed(range(len(self._saved)))):
            dx = gb["g"][i % 2]
            self.backward_application(self._saved[r], g, dx, accumulate or i > 0, stream)
            g = dx
        return g

    def flops(self, T, R):
        return 2.0 * T * self.d * (self.nqkv + self.d + 2 * self.H) * R

    def flops_bwd(self, T, R):
        """Contractions of backward(): per application the MLP's four GEMMs
        (2*T*d*H each) and the O and Q projections' two each (2*T*d*d)."""
        return (8.0 * T * self.d * self.H + 8.0 * T * self.d * self.d) * R


class HeadMlpStep:
    """One QAT training step of a tied int8 head over an int6 ReLU^2 MLP:
        quantize (every step: the weights change between steps)
        Z = MLP(X); logits = Z Wemb^T
        dZ = dLogits Wemb_q; dWemb = dLogits^T Z; MLP backward -> dX, dWfc, dWproj
    """

    def __init__(self, Wemb, Wfc, Wproj, T, head_bits=8, mlp_bits=6, act="relu2"):
        dev = Wemb.device
        self.W = (Wemb, Wfc, Wproj)
        self.vocab, self.d = Wemb.shape
        self.H = Wfc.shape[0]
        self.T = T
        self.head_bits, self.mlp_bits = head_bits, mlp_bits
        self.act = act
        bf = torch.bfloat16
        e = lambda *s, dt=bf: torch.empty(s, dtype=dt, device=dev)
        self.q = [qat.QWeight(e(*w.shape), e(w.shape[0], dt=torch.float32), None, b)
                  for w, b in ((Wemb, head_bits), (Wfc, mlp_bits), (Wproj, mlp_bits))]
        self.pre, self.h = e(T, self.H), e(T, self.H)
        self.Z, self.logits, self.dZ, self.dX = e(T, self.d), e(T, self.vocab), e(T, self.d), e(T, self.d)
        self.dWemb = e(self.vocab, self.d, dt=torch.float32)
        self.dWfc = e(self.H, self.d, dt=torch.float32)
        self.dWproj = e(self.d, self.H, dt=torch.float32)
        ws = qat.workspace_size(qat.QAT_OP_MLP_BWD, self.d, self.H, T, False)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)

    def quantize(self, stream=None):
        """All three weights' operands in one launch."""
        qat.qat_quantize_weights_batch([(w, q.bits, q.scales, None, q.operand)
                                        for w, q in zip(self.W, self.q)], stream)

    def forward(self, X, stream=None):
        qe, qf, qp = self.q
        qat.qat_mlp_fwd(X, self.Z, self.mlp_bits, self.d, self.H, qfc=qf, qproj=qp,
                        pre_save=self.pre, h_save=self.h, stream=stream, act=self.act)
        qat.qat_linear_fwd(self.Z, self.logits, self.head_bits, qw=qe, stream=stream)

    def backward(self, X, dLogits, stream=None, on_head_grad=None):
        """on_head_grad(): called once the head's backward is queued (its dWemb
        is then complete in stream order), before the MLP backward."""
        qe, qf, qp = self.q
        qat.qat_linear_bwd(self.Z, dLogits, self.head_bits, qw=qe, dX=self.dZ, dW=self.dWemb,
                           stream=stream)
        if on_head_grad is not None:
            on_head_grad()
        qat.qat_mlp_bwd(X, self.pre, self.h, self.dZ, self.mlp_bits, self.d, self.H, qfc=qf,
                        qproj=qp, dX=self.dX, dWfc=self.dWfc, dWproj=self.dWproj,
                        workspace=self.ws, stream=stream, act=self.act)

    def step(self, X, dLogits, stream=None, on_head_grad=None):
        self.quantize(stream)
        self.forward(X, stream)
        self.backward(X, dLogits, stream, on_head_grad)

    def grads(self):
        return [self.dWemb, self.dWfc, self.dWproj]

    def flops_per_token(self):
        # forward + two backward GEMMs for the head and for each MLP linear
        return 3 * 2.0 * self.d * (self.vocab + 2 * self.H)
