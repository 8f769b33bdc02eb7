"""Oracle of the looped nGPT forward pass (TEST INFRASTRUCTURE, see package
docstring).  float64 NumPy; every function cites the passage it follows.

Passages (page title, section):
  [LOOP]  "Dory1.0-4B: 循环归一化 GPT" (paper summary), 核心方法:
          s0 = x, u_t = N(s_{t-1} + x), s_t = N(F_theta(u_t)), t = 1..k;
          effective depth 32 + 40k sublayers; recurrent parameters shared.
  [NGPT]  same page, 前置知识 / nGPT: s <- N((1-alpha) s + alpha sublayer(s)),
          per-channel alpha.
  [ARCH]  "Dory1.0-4B: A Looped Normalized-GPT" (paperlayer summary), §2
          Architecture: normalised sublayer output blended with the
          normalised residual by learned per-channel weights, then
          normalised; gated attention outputs and SwiGLU activations are
          L2-normalised before their output projections; query-key scale and
          logit-scale parameters.
  [ATTN]  paper summary, 技术新颖性: 3:1 sliding-window (W=1024, RoPE base 1e4)
          to full attention (RoPE base 1e7), GQA 16 query / 4 KV heads,
          input-dependent sigmoid output gate.
  [KV]    paperlayer §6.1 Last-Loop KV Caching: each recurrent layer's cache
          is overwritten at every loop; earlier-loop queries attend to
          final-loop entries for prior tokens.  MXFP8 explainer page,
          "循环 + KV 缓存" section: one cache per recurrent attention layer.
"""
import numpy as np

DT = np.float64


def l2n(v, axis=-1):
    """N(v) = v / max(||v||_2, 1e-12) over ``axis`` [NGPT]."""
    v = np.asarray(v, dtype=DT)
    n = np.sqrt(np.sum(v * v, axis=axis, keepdims=True))
    return v / np.maximum(n, 1e-12)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    return x * sigmoid(x)


def rope(v, pos, theta):
    """Rotary position embedding, rotate-half pairing (dims i and i + h/2).

    v: [..., T, h]; pos: [T] absolute token positions.  Frequencies
    theta^(-2i/h), i < h/2, angles in float64.  The pages fix only the base
    per attention type [ATTN]; the pairing convention is a reading.
    """
    v = np.asarray(v, dtype=DT)
    h = v.shape[-1]
    half = h // 2
    inv = theta ** (-(2.0 * np.arange(half, dtype=DT)) / h)
    ang = np.asarray(pos, dtype=DT)[:, None] * inv[None, :]      # [T, half]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def attention(q, K, V, q_pos, k_pos, window, scale):
    """Causal softmax attention with GQA, vectorised over query positions.

    q: [Hq, T, h]; K, V: [Hkv, P, h]; q_pos [T]; k_pos [P].
    Query head j reads KV head j // (Hq / Hkv) (contiguous groups).
    Visible keys: k_pos <= q_pos, and for a sliding window W additionally
    k_pos > q_pos - W (W keys including the query's own) [ATTN].
    """
    Hq, T, h = q.shape
    Hkv = K.shape[0]
    group = Hq // Hkv
    qp = np.asarray(q_pos)[:, None]
    kp = np.asarray(k_pos)[None, :]
    mask = kp <= qp
    if window:
        mask &= kp > qp - window
    out = np.empty((Hq, T, V.shape[-1]), dtype=DT)
    for j in range(Hq):
        kv = j // group
        sc = scale * (q[j] @ K[kv].T)
        sc = np.where(mask, sc, -np.inf)
        sc = sc - sc.max(axis=1, keepdims=True)
        e = np.exp(sc)
        e = e / e.sum(axis=1, keepdims=True)
        out[j] = e @ V[kv]
    return out


def attention_bruteforce(q, K, V, q_pos, k_pos, window, scale):
    """Same definition as ``attention`` written as scalar loops (tiny inputs)."""
    Hq, T, h = q.shape
    group = Hq // K.shape[0]
    out = np.zeros((Hq, T, V.shape[-1]), dtype=DT)
    for j in range(Hq):
        kv = j // group
        for t in range(T):
            vis = [i for i in range(len(k_pos))
                   if k_pos[i] <= q_pos[t]
                   and (not window or k_pos[i] > q_pos[t] - window)]
            logits = [scale * float(np.dot(q[j, t], K[kv, i])) for i in vis]
            mx = max(logits)
            w = [np.exp(x - mx) for x in logits]
            tot = sum(w)
            for wi, i in zip(w, vis):
                out[j, t] += (wi / tot) * V[kv, i]
    return out


def ngpt_update(s, h, alpha):
    """s <- N(s + alpha * (N(h) - s)) = N((1-alpha) s + alpha N(h)) [NGPT, ARCH]."""
    return l2n(s + alpha * (l2n(h) - s))


def swiglu(gate, up):
    """m = N(silu(gate) * up), normalised before the down projection [ARCH]."""
    return l2n(silu(gate) * up)


def greedy(z):
    """argmax over the last axis; numpy returns the lowest index on ties."""
    return np.argmax(z, axis=-1)


class Model:
    """Looped nGPT over B sequences of equal length, with its KV cache.

    weights: {name: array}; BF16 matrices as uint16 bit patterns (widened
    exactly), vectors as float.  kv_mode: "per_loop" (one cache per loop per
    recurrent attention layer; the call's loop count is fixed for the life of
    the cache) or "last_loop" (one cache per recurrent attention layer,
    overwritten by every loop) [KV].  Input and output blocks always have one
    cache each.

    The cache stores every position (no ring); the sliding window is applied
    as a mask when reading.  Write/read order inside one attention sublayer:
    all K/V of the call's tokens are stored in the chosen slot first, then
    every query reads whatever each visible position holds.  In last_loop
    mode a call's own tokens therefore see same-loop entries while earlier
    tokens hold their final-loop values [KV].
    """

    def __init__(self, shape, weights, batch=1, kv_mode="per_loop",
                 trace=None, keep_decoded=None):
        if kv_mode not in ("per_loop", "last_loop"):
            raise ValueError(kv_mode)
        self.shape, self.w, self.B, self.kv_mode = shape, weights, batch, kv_mode
        self.trace = trace
        self.n_ctx = 0
        self.n_loops_fixed = None
        self.cache = {}
        self.sublayers = 0
        if keep_decoded is None:
            keep_decoded = shape.params_per_block() * shape.n_blocks < 5e7
        self._keep = keep_decoded
        self._dec = {}

    # ---- weights -------------------------------------------------------
    def W(self, name):
        """Weight `name` in float64: BF16 bits widened exactly, or a quantised
        matrix (name.q / name.s [/ name.t]) decoded by oracle.quant: MXFP8
        when there is no tensor scale, NVFP4 (with its f32 tensor scale)
        otherwise."""
        if name in self._dec:
            return self._dec[name]
        if name not in self.w and name + ".q" in self.w:
            from . import quant
            q, sc = self.w[name + ".q"], self.w[name + ".s"]
            if name + ".t" in self.w:
                out = quant.dequant_nvfp4(q, sc, float(self.w[name + ".t"][0]))
            else:
                out = quant.dequant_mxfp8(q, sc)
            out = np.asarray(out, dtype=DT)
            if self._keep:
                self._dec[name] = out
            return out
        t = self.w[name]
        if isinstance(t, np.ndarray) and t.dtype == np.uint16:
            out = (t.astype(np.uint32) << 16).view(np.float32).astype(DT)
        else:
            out = np.asarray(t, dtype=DT)
        if self._keep:
            self._dec[name] = out
        return out

    def rows(self, name, idx):
        t = self.w[name][np.asarray(idx)]
        if t.dtype == np.uint16:
            return (t.astype(np.uint32) << 16).view(np.float32).astype(DT)
        return np.asarray(t, dtype=DT)

    def _emit(self, kind, i, s):
        if self.trace is not None:
            self.trace(kind, i, s)

    # ---- cache ---------------------------------------------------------
    def slot_of(self, i, t):
        gin, grec, gout = self.shape.block_groups()
        if i in grec and self.kv_mode == "per_loop":
            return t
        return 0

    def slot_arrays(self, i, slot, need):
        sh = self.shape
        key = (i, slot)
        if key not in self.cache or self.cache[key][0].shape[2] < need:
            K = np.zeros((self.B, sh.n_kv_heads, need, sh.head_dim), DT)
            V = np.zeros_like(K)
            if key in self.cache:
                old = self.cache[key][0].shape[2]
                K[:, :, :old] = self.cache[key][0]
                V[:, :, :old] = self.cache[key][1]
            self.cache[key] = (K, V)
        return self.cache[key]

    def kv_slots(self):
        """Distinct (block, slot) caches in use."""
        return sorted(self.cache)

    # ---- sublayers -----------------------------------------------------
    def attn_sublayer(self, i, s, pos, slot):
        sh = self.shape
        B, T, d = s.shape
        Hq, Hkv, h = sh.n_q_heads, sh.n_kv_heads, sh.head_dim
        qd, kvd = sh.qdim, sh.kvdim
        proj = s @ self.W(f"blk{i}.w_qkvg").T
        q = proj[..., :qd].reshape(B, T, Hq, h).transpose(0, 2, 1, 3)
        k = proj[..., qd:qd + kvd].reshape(B, T, Hkv, h).transpose(0, 2, 1, 3)
        v = proj[..., qd + kvd:qd + 2 * kvd].reshape(B, T, Hkv, h
                                                     ).transpose(0, 2, 1, 3)
        g = proj[..., qd + 2 * kvd:]
        full = sh.layer_types[i] == 1
        theta = sh.rope_theta_full if full else sh.rope_theta_swa
        s_q = self.W(f"blk{i}.s_q")[None, :, None, :]
        s_k = self.W(f"blk{i}.s_k")[None, :, None, :]
        q = s_q * l2n(rope(q, pos, theta))
        k = s_k * l2n(rope(k, pos, theta))
        end = int(pos[-1]) + 1
        K, V = self.slot_arrays(i, slot, end)
        K[:, :, pos] = k
        V[:, :, pos] = v
        kpos = np.arange(end)
        window = 0 if full else sh.swa_window
        o = np.stack([attention(q[b], K[b, :, :end], V[b, :, :end], pos, kpos,
                                window, np.sqrt(h)) for b in range(B)])
        o = o.transpose(0, 2, 1, 3).reshape(B, T, qd)
        a = l2n(sigmoid(g) * o)
        hA = a @ self.W(f"blk{i}.w_o").T
        s = ngpt_update(s, hA, self.W(f"blk{i}.alpha_a"))
        self.sublayers += 1
        self._emit("attn", i, s)
        return s

    def mlp_sublayer(self, i, s):
        F = self.shape.ffn
        gu = s @ self.W(f"blk{i}.w_gu").T
        m = swiglu(gu[..., :F], gu[..., F:])
        hM = m @ self.W(f"blk{i}.w_down").T
        s = ngpt_update(s, hM, self.W(f"blk{i}.alpha_m"))
        self.sublayers += 1
        self._emit("mlp", i, s)
        return s

    def block(self, i, s, pos, t):
        s = self.attn_sublayer(i, s, pos, self.slot_of(i, t))
        return self.mlp_sublayer(i, s)

    # ---- forward -------------------------------------------------------
    def forward(self, tokens, n_loops, all_logits=False):
        """Run the call's tokens [B, T] through the looped stack [LOOP].

        Returns logits [B, T, V] (all_logits) or [B, 1, V] for the last
        position: z = s_z * (W_lm s) [ARCH].
        """
        if n_loops < 1:
            raise ValueError("n_loops must be >= 1")
        if self.kv_mode == "per_loop":
            if self.n_loops_fixed is None:
                self.n_loops_fixed = n_loops
            elif self.n_loops_fixed != n_loops:
                raise ValueError("per_loop cache bound to another loop count")
        tokens = np.asarray(tokens).reshape(self.B, -1)
        T = tokens.shape[1]
        pos = np.arange(self.n_ctx, self.n_ctx + T)
        gin, grec, gout = self.shape.block_groups()
        x = l2n(self.rows("embed", tokens))
        self._emit("embed", -1, x)
        s = x
        for i in gin:
            s = self.block(i, s, pos, 0)
        x = s                                       # input-block output
        for t in range(1, n_loops + 1):
            s = l2n(s + x)                          # u_t = N(s_{t-1} + x)
            self._emit("loop_in", t, s)
            for i in grec:
                s = self.block(i, s, pos, t)
            s = l2n(s)                              # s_t = N(F(u_t))
            self._emit("loop_out", t, s)
        for i in gout:
            s = self.block(i, s, pos, 0)
        self.n_ctx += T
        self.last_state = s
        sel = s if all_logits else s[:, -1:]
        return self.lm_head(sel)

    def lm_head(self, s):
        V = self.shape.vocab
        sz = self.W("s_z")
        z = np.empty(s.shape[:-1] + (V,), dtype=DT)
        step = 16384
        for r0 in range(0, V, step):
            r1 = min(V, r0 + step)
            Wl = self.rows("lm_head", np.arange(r0, r1))
            z[..., r0:r1] = sz[r0:r1] * (s @ Wl.T)
        return z

    prefill = forward

    def decode_step(self, tokens, n_loops):
        """One token per sequence; returns logits [B, V]."""
        return self.forward(np.asarray(tokens).reshape(self.B, 1),
                            n_loops)[:, 0]
