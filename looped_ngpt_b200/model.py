"""Python binding of the C ABI: argument marshalling around libdory.so.

PyTorch provides device memory and streams only; every step of the forward
pass runs in the library's CUDA kernels.  Names follow the C entry points:
``DoryModel.prefill`` -> ``dory_prefill``, ``DoryModel.decode_step`` ->
``dory_decode_step``, and so on.
"""
import ctypes

import numpy as np
import torch

from . import _lib
from ._lib import DoryConfig, DoryTensor, check, KV_MODES


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def to_device(arr, device):
    """numpy array -> device tensor (uint16 arrays are BF16 bit patterns)."""
    a = np.ascontiguousarray(arr)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    if a.dtype == np.uint8:
        return torch.from_numpy(a).to(device)
    return torch.from_numpy(a.astype(np.float32)).to(device)


class KVCache:
    """A caller-owned device buffer bound as a dory_cache."""

    def __init__(self, model, batch, max_ctx, max_chunk, max_loops, kv_mode,
                 stream=None):
        self.model = model
        self.batch, self.max_ctx, self.max_chunk = batch, max_ctx, max_chunk
        self.kv_mode = kv_mode
        lib = _lib.load()
        nbytes = ctypes.c_int64()
        check("dory_kv_cache_bytes", lib.dory_kv_cache_bytes(
            model.handle, batch, max_ctx, max_chunk, max_loops,
            KV_MODES[kv_mode], ctypes.byref(nbytes)))
        self.nbytes = nbytes.value
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8,
                               device=model.device)
        h = ctypes.c_void_p()
        check("dory_kv_cache_bind", lib.dory_kv_cache_bind(
            model.handle, ctypes.c_void_p(self.buf.data_ptr()), self.nbytes,
            batch, max_ctx, max_chunk, max_loops, KV_MODES[kv_mode],
            _stream_ptr(stream), ctypes.byref(h)))
        self.handle = h

    def length(self):
        n = ctypes.c_int()
        check("dory_cache_length",
              _lib.load().dory_cache_length(self.handle, ctypes.byref(n)))
        return n.value

    def fill_synthetic(self, n_ctx, seed=2, stream=None):
        """dory_cache_fill_synthetic: n_ctx seeded synthetic tokens per row."""
        check("dory_cache_fill_synthetic",
              _lib.load().dory_cache_fill_synthetic(
                  self.model.handle, self.handle, n_ctx, seed,
                  _stream_ptr(stream)))

    def copy_prefix_from(self, src, src_b, n_tokens, stream=None):
        """dory_cache_copy_prefix: every sequence of this cache takes the
        first n_tokens positions of sequence src_b of `src`."""
        check("dory_cache_copy_prefix", _lib.load().dory_cache_copy_prefix(
            self.model.handle, self.handle, src.handle, src_b, n_tokens,
            _stream_ptr(stream)))

    def reset(self, stream=None):
        check("dory_cache_reset",
              _lib.load().dory_cache_reset(self.handle, _stream_ptr(stream)))

    def __del__(self):
        if getattr(self, "handle", None) and _lib._lib is not None:
            _lib._lib.dory_cache_free(self.handle)
            self.handle = None


class DoryModel:
    """Weights of one looped nGPT resident in HBM, bound to libdory."""

    def __init__(self, shape, weights, device="cuda"):
        self.shape = shape
        self.device = torch.device(device)
        lib = _lib.load()
        self.tensors = {n: (t if isinstance(t, torch.Tensor)
                            else to_device(t, self.device))
                        for n, t in weights.items()}
        self._names = [n.encode() for n in self.tensors]
        arr = (DoryTensor * len(self.tensors))()
        for i, (n, t) in enumerate(self.tensors.items()):
            arr[i] = DoryTensor(self._names[i], t.data_ptr(),
                                t.numel() * t.element_size())
        # weight format of the block projections, from the tensor names
        self.wfmt = 0
        if "blk0.w_qkvg.t" in self.tensors:
            self.wfmt = 2
        elif "blk0.w_qkvg.q" in self.tensors:
            self.wfmt = 1
        lt = (ctypes.c_uint8 * shape.n_blocks)(*shape.layer_types)
        cfg = DoryConfig(shape.d, shape.n_q_heads, shape.n_kv_heads,
                         shape.head_dim, shape.ffn, shape.vocab, shape.n_in,
                         shape.n_rec, shape.n_out, lt, shape.swa_window,
                         shape.rope_theta_swa, shape.rope_theta_full,
                         self.wfmt)
        h = ctypes.c_void_p()
        check("dory_init_weights", lib.dory_init_weights(
            ctypes.byref(cfg), arr, len(self.tensors), ctypes.byref(h)))
        self.handle = h

    def weight_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.tensors.values())

    # ---- buffers ---------------------------------------------------------
    def new_cache(self, batch, max_ctx, max_chunk, kv_mode="last_loop",
                  max_loops=4, stream=None):
        return KVCache(self, batch, max_ctx, max_chunk, max_loops, kv_mode,
                       stream)

    def workspace(self, batch, max_chunk):
        n = ctypes.c_int64()
        check("dory_workspace_bytes", _lib.load().dory_workspace_bytes(
            self.handle, batch, max_chunk, ctypes.byref(n)))
        return torch.empty(n.value, dtype=torch.uint8, device=self.device)

    # ---- calls -----------------------------------------------------------
    def prefill(self, cache, tokens, n_loops, ws, logits_all=False,
                logits=None, argmax=None, stream=None):
        """dory_prefill on device tokens int32 [B, T]; returns (logits, argmax)."""
        B, T = tokens.shape
        V = self.shape.vocab
        if logits is None:
            logits = torch.empty((B, T, V) if logits_all else (B, V),
                                 dtype=torch.float32, device=self.device)
        if argmax is None:
            argmax = torch.empty((B, T) if logits_all else (B,),
                                 dtype=torch.int32, device=self.device)
        check("dory_prefill", _lib.load().dory_prefill(
            self.handle, cache.handle, ctypes.c_void_p(tokens.data_ptr()), B, T,
            n_loops, KV_MODES[cache.kv_mode], 1 if logits_all else 0,
            ctypes.c_void_p(logits.data_ptr()),
            ctypes.c_void_p(argmax.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
            ws.numel(), _stream_ptr(stream)))
        return logits, argmax

    def decode_step(self, cache, tokens, n_loops, ws, logits=None,
                    argmax=None, want_logits=True, stream=None):
        """dory_decode_step on device tokens int32 [B]; returns (logits, argmax)."""
        B = tokens.shape[0]
        # Fixed per-cache token/output buffers keep the pointers of repeated
        # steps identical, so the library can replay its captured graph.
        if getattr(cache, "_dec_bufs", None) is None:
            cache._dec_bufs = (
                torch.empty((B,), dtype=torch.int32, device=self.device),
                torch.empty((B, self.shape.vocab), dtype=torch.float32,
                            device=self.device),
                torch.empty((B,), dtype=torch.int32, device=self.device))
        tok_buf, lg_buf, am_buf = cache._dec_bufs
        if tokens.data_ptr() != tok_buf.data_ptr():
            tok_buf.copy_(tokens.reshape(B), non_blocking=True)
        tokens = tok_buf
        if logits is None and want_logits:
            logits = lg_buf
        if argmax is None:
            argmax = am_buf
        check("dory_decode_step", _lib.load().dory_decode_step(
            self.handle, cache.handle, ctypes.c_void_p(tokens.data_ptr()), B,
            n_loops, KV_MODES[cache.kv_mode],
            ctypes.c_void_p(logits.data_ptr() if logits is not None else 0),
            ctypes.c_void_p(argmax.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
            ws.numel(), _stream_ptr(stream)))
        return logits, argmax

    def prefill_mixed(self, cache, tokens, row_loops, ws, logits_all=False,
                      stream=None):
        """dory_prefill_mixed: sequence b runs row_loops[b] loops (device
        int32 [B]); returns (logits, argmax)."""
        B, T = tokens.shape
        V = self.shape.vocab
        logits = torch.empty((B, T, V) if logits_all else (B, V),
                             dtype=torch.float32, device=self.device)
        argmax = torch.empty((B, T) if logits_all else (B,), dtype=torch.int32,
                             device=self.device)
        check("dory_prefill_mixed", _lib.load().dory_prefill_mixed(
            self.handle, cache.handle, ctypes.c_void_p(tokens.data_ptr()), B, T,
            ctypes.c_void_p(row_loops.data_ptr()), int(row_loops.max()),
            KV_MODES[cache.kv_mode], 1 if logits_all else 0,
            ctypes.c_void_p(logits.data_ptr()),
            ctypes.c_void_p(argmax.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
            ws.numel(), _stream_ptr(stream)))
        return logits, argmax

    def decode_step_mixed(self, cache, tokens, row_loops, max_loops, ws,
                          stream=None):
        """dory_decode_step_mixed on device tokens int32 [B] and per-row loop
        counts row_loops int32 [B]; returns (logits, argmax)."""
        B = tokens.shape[0]
        if getattr(cache, "_mix_bufs", None) is None:
            cache._mix_bufs = (
                torch.empty((B,), dtype=torch.int32, device=self.device),
                torch.empty((B, self.shape.vocab), dtype=torch.float32,
                            device=self.device),
                torch.empty((B,), dtype=torch.int32, device=self.device),
                torch.empty((B,), dtype=torch.int32, device=self.device))
        tok_buf, lg_buf, am_buf, rl_buf = cache._mix_bufs
        tok_buf.copy_(tokens.reshape(B), non_blocking=True)
        rl_buf.copy_(row_loops.reshape(B), non_blocking=True)
        check("dory_decode_step_mixed", _lib.load().dory_decode_step_mixed(
            self.handle, cache.handle, ctypes.c_void_p(tok_buf.data_ptr()), B,
            ctypes.c_void_p(rl_buf.data_ptr()), max_loops,
            KV_MODES[cache.kv_mode], ctypes.c_void_p(lg_buf.data_ptr()),
            ctypes.c_void_p(am_buf.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
            ws.numel(), _stream_ptr(stream)))
        return lg_buf, am_buf

    def spec_workspace(self, batch, gamma):
        n = ctypes.c_int64()
        check("dory_spec_workspace_bytes", _lib.load().dory_spec_workspace_bytes(
            self.handle, batch, gamma, ctypes.byref(n)))
        return torch.empty(n.value, dtype=torch.uint8, device=self.device)

    def spec_decode_step(self, cache, last, gamma, k_draft, k_verify, ws,
                         temperature=0.0, uniform=None, out=None, stream=None):
        """dory_spec_decode_step: draft gamma tokens at k_draft loops, verify
        at k_verify; returns (tokens int32 [B, gamma + 1], n emitted)."""
        B = last.shape[0]
        if out is None:
            out = torch.empty((B, gamma + 1), dtype=torch.int32,
                              device=self.device)
        n = ctypes.c_int()
        check("dory_spec_decode_step", _lib.load().dory_spec_decode_step(
            self.handle, cache.handle, ctypes.c_void_p(last.data_ptr()), B,
            gamma, k_draft, k_verify, float(temperature),
            ctypes.c_void_p(uniform.data_ptr() if uniform is not None else 0),
            ctypes.c_void_p(out.data_ptr()), ctypes.byref(n),
            ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream_ptr(stream)))
        return out, n.value

    def copy_state(self, ws, B, T, logits_all=False, stream=None):
        """dory_copy_state: final residual state of the last call."""
        rows = B * T if logits_all else B
        out = torch.empty((rows, self.shape.d), dtype=torch.float32,
                          device=self.device)
        check("dory_copy_state", _lib.load().dory_copy_state(
            self.handle, ctypes.c_void_p(ws.data_ptr()), B, T,
            1 if logits_all else 0, ctypes.c_void_p(out.data_ptr()),
            _stream_ptr(stream)))
        return out

    def profile(self, on=True):
        """dory_profile_enable: per-kernel CUDA-event timing of later calls."""
        check("dory_profile_enable",
              _lib.load().dory_profile_enable(self.handle, 1 if on else 0))

    def profile_read(self, stream=None):
        """dory_profile_read -> {kernel class: {launches, ms, bytes, flops}}."""
        arr = (_lib.DoryKernelStat * 64)()
        n = ctypes.c_int()
        check("dory_profile_read", _lib.load().dory_profile_read(
            self.handle, arr, 64, ctypes.byref(n), _stream_ptr(stream)))
        return {arr[i].name.decode(): dict(launches=arr[i].launches,
                                           ms=arr[i].total_ms,
                                           bytes=arr[i].bytes,
                                           flops=arr[i].flops)
                for i in range(n.value)}

    def debug_dequant(self, tensor, row0, nrows, K, stream=None):
        """dory_debug_dequant: f32 [nrows, K] decoded weights."""
        out = torch.empty((nrows, K), dtype=torch.float32, device=self.device)
        check("dory_debug_dequant", _lib.load().dory_debug_dequant(
            self.handle, tensor.encode(), row0, nrows,
            ctypes.c_void_p(out.data_ptr()), _stream_ptr(stream)))
        return out

    def debug_gemv(self, tensor, x, stream=None):
        """dory_debug_gemv: the production decode GEMV of block projection
        `tensor` on bf16 rows x [B, K]; returns the f32 partial slabs
        [n, B, N] (their sum is the product)."""
        B, K = x.shape
        N = {"w_qkvg": self.shape.qkvg_rows, "w_o": self.shape.d,
             "w_gu": 2 * self.shape.ffn, "w_down": self.shape.d}[
                 tensor.split(".", 1)[1]]
        cap = 16
        out = torch.empty((cap, B, N), dtype=torch.float32, device=self.device)
        n = ctypes.c_int()
        check("dory_debug_gemv", _lib.load().dory_debug_gemv(
            self.handle, tensor.encode(), ctypes.c_void_p(x.data_ptr()), B,
            ctypes.c_void_p(out.data_ptr()), cap, ctypes.byref(n),
            _stream_ptr(stream)))
        return out[:n.value]

    def sync_status(self, stream=None):
        return _lib.load().dory_sync_status(self.handle, _stream_ptr(stream))

    def __del__(self):
        if getattr(self, "handle", None) and _lib._lib is not None:
            _lib._lib.dory_free(self.handle)
            self.handle = None
