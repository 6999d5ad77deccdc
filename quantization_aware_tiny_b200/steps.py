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

    def _train_buffers(self, T, R, device):
        """Activations and gradients of every application, stacked [R, T, .]
        so that each weight gradient is one GEMM over all R * T token uses:
        states [R+1, T, d] (state 0 is the input, state r+1 the output of
        application r), qkv, x1, pre, h; the gradient's g [R, T, d] (g[r] =
        dL/d output of application r), dx1, dq [R, T, d], dpre [R, T, H].
        They, and the weight gradients dWqkv, dWo, dWfc, dWproj, are allocated
        again when T or R changes: accumulate=True carries gradients across
        calls of the same T and R only."""
        key = (T, R)
        if getattr(self, "_tkey", None) != key:
            bf, f32 = torch.bfloat16, torch.float32
            e = lambda *sh, dt=bf: torch.empty(sh, dtype=dt, device=device)
            d, H = self.d, self.H
            self._tb = {"states": e(R + 1, T, d), "qkv": e(R, T, self.nqkv), "x1": e(R, T, d),
                        "pre": e(R, T, H), "h": e(R, T, H), "g": e(R, T, d), "dx1": e(R, T, d),
                        "dq": e(R, T, d), "dpre": e(R, T, H), "dX": e(T, d)}
            self.dWqkv = e(self.nqkv, d, dt=f32)
            self.dWo = e(d, d, dt=f32)
            self.dWfc = e(H, d, dt=f32)
            self.dWproj = e(d, H, dt=f32)
            self._tkey = key
        return self._tb

    def forward_train(self, x, R, stream=None, noise=None):
        """The forward of forward() for training: x [T,d] bf16 is left as it is
        (copied in as state 0) and every application's activations are kept
        for backward().  Returns the output state of the last application (a
        buffer the core owns)."""
        T = x.shape[0]
        tb = self._train_buffers(T, R, x.device)
        apps = self._ops_for_noise(noise, R, stream) if noise is not None else \
            [(self.q_qkv, self.q_o, self.q_fc, self.q_proj)] * R
        st = tb["states"]
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
            st[0].copy_(x)
        for r in range(R):
            q_qkv, q_o, q_fc, q_proj = apps[r]
            qat.qat_linear_fwd(st[r], tb["qkv"][r], self.bits, qw=q_qkv, stream=stream)
            qat.qat_linear_fwd(tb["qkv"][r], tb["x1"][r], self.bits, qw=q_o, ldx=self.nqkv, T=T,
                               residual=st[r], stream=stream)
            qat.qat_mlp_fwd(tb["x1"][r], st[r + 1], self.bits, self.d, self.H, qfc=q_fc,
                            qproj=q_proj, residual=tb["x1"][r], pre_save=tb["pre"][r],
                            h_save=tb["h"][r], stream=stream, act=self.act)
        self._apps, self._R = apps, R
        return st[R]

    def _saved(self, r):
        """Application r's kept activations and operands (for backward_application)."""
        tb = self._tb
        return {"x": tb["states"][r], "qkv": tb["qkv"][r], "x1": tb["x1"][r], "pre": tb["pre"][r],
                "h": tb["h"][r], "ops": self._apps[r]}

    def _dx_chain(self, s, g, dx1, dq, dpre, dx, stream):
        """The gradient's chain through one application (no weight gradients):
            dpre = (g Wproj) * act'(pre) ; dx1 = g + dpre Wfc   (qat_mlp_bwd)
            dq   = dx1 Wo                                       (qat_linear_bwd)
            dx   = dx1 + dq Wq                                  (qat_linear_bwd)"""
        q_qkv, q_o, q_fc, q_proj = s["ops"]
        d = self.d
        qat.qat_mlp_bwd(s["x1"], s["pre"], s["h"], g, self.bits, d, self.H, qfc=q_fc,
                        qproj=q_proj, dX=dx1, dX_residual=g, dpre_save=dpre, stream=stream,
                        act=self.act)
        qat.qat_linear_bwd(None, dx1, self.bits, qw=q_o, dX=dq, stream=stream)
        q_q = qat.QWeight(q_qkv.operand[:d], None, None, self.bits)
        qat.qat_linear_bwd(None, dq, self.bits, qw=q_q, dX=dx, dX_residual=dx1, stream=stream)

    def _weight_grads(self, x, qkv, x1, h, g, dx1, dq, dpre, accumulate, stream):
        """The four weight gradients from token-stacked operands (one GEMM each,
        the reduction over every token of every application given):
            dWproj (+)= g^T h ; dWfc (+)= dpre^T x1 ; dWo (+)= dx1^T q ;
            dWqkv[:d] (+)= dq^T x ; dWqkv[d:] = 0 unless accumulating
        (k and v do not reach the output with attention left out)."""
        d, H = self.d, self.H
        qat.qat_linear_bwd(h, g, self.bits, dW=self.dWproj, N=d, K=H,
                           accumulate_dW=accumulate, stream=stream)
        qat.qat_linear_bwd(x1, dpre, self.bits, dW=self.dWfc, N=H, K=d,
                           accumulate_dW=accumulate, stream=stream)
        qat.qat_linear_bwd(qkv, dx1, self.bits, dW=self.dWo, N=d, K=d, ldx=self.nqkv,
                           accumulate_dW=accumulate, stream=stream)
        qat.qat_linear_bwd(x, dq, self.bits, dW=self.dWqkv[:d], N=d, K=d,
                           accumulate_dW=accumulate, stream=stream)
        if not accumulate:  # T = 0 call: zeroes the k|v rows of dWqkv
            qat.qat_linear_bwd(None, dq[:0], self.bits, dW=self.dWqkv[d:],
                               N=self.nqkv - d, K=d, stream=stream)

    def backward_application(self, s, g, dx, accumulate, stream=None):
        """STE backward of one application from its activations s (x, qkv, x1,
        pre, h and its operands) and g = dL/d out: dL/dx into dx, and that
        application's weight gradients written into (or, accumulate, added to)
        dWqkv, dWo, dWfc, dWproj."""
        T = g.shape[0]
        if getattr(self, "_tkey", None) is None or self._tkey[0] != T:
            self._train_buffers(T, 1, g.device)
        tb = self._tb
        dx1, dq, dpre = tb["dx1"][0], tb["dq"][0], tb["dpre"][0]
        self._dx_chain(s, g, dx1, dq, dpre, dx, stream)
        self._weight_grads(s["x"], s["qkv"], s["x1"], s["h"], g, dx1, dq, dpre, accumulate, stream)

    def backward(self, dY, stream=None, accumulate=False):
        """Backward through the applications of the last forward_train, in
        reverse, the shared weights' gradients summed over the R uses (P1
        "税 1").  The gradient's chain runs application by application (4
        GEMMs each, the per-application gradients kept); then each weight's
        gradient is ONE GEMM whose reduction runs over the R * T token uses
        (the stacked activations and gradients), instead of R accumulating
        ones.  dY = dL/d(output state) [T,d] bf16.  Returns dL/dx (a buffer
        the core owns); weight gradients in dWqkv, dWo, dWfc, dWproj (fp32,
        overwritten, or added to with accumulate=True)."""
        R, tb = self._R, self._tb
        T = dY.shape[0]
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
            tb["g"][R - 1].copy_(dY)
        for r in reversed(range(R)):
            dx = tb["g"][r - 1] if r > 0 else tb["dX"]
            self._dx_chain(self._saved(r), tb["g"][r], tb["dx1"][r], tb["dq"][r], tb["dpre"][r],
                           dx, stream)
        flat = lambda a: a.reshape(R * T, a.shape[-1])
        self._weight_grads(flat(tb["states"][:R]), flat(tb["qkv"]), flat(tb["x1"]), flat(tb["h"]),
                           flat(tb["g"]), flat(tb["dx1"]), flat(tb["dq"]), flat(tb["dpre"]),
                           accumulate, stream)
        return tb["dX"]

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
