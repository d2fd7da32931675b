"""SAGA + Atop-N single-token decode attention on B200 (sm_100a).

Thin Python binding over the C ABI of ``libsaga.so`` (declared in
``include/saga.h``).  Every step of the computation runs in the library's CUDA
kernels; this module only checks tensor shapes, dtypes and devices and passes
raw pointers and the current CUDA stream.  torch supplies device memory and
streams.  There is no CPU fallback: if the library is missing, or a call fails,
an exception is raised.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import SagaError, load  # noqa: F401

__all__ = ["SagaDecoder", "SagaError", "load", "combine_noalloc"]


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t: torch.Tensor, name: str, dtype, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device == "cuda" and not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if device == "cpu" and t.is_cuda:
        raise ValueError(f"{name} must be in host memory")


class SagaDecoder:
    """A handle of the library: fixed head layout and maximum sizes, one workspace.

    head_dim_v (default head_dim) is the value and output width: keys may be
    narrower (or wider) than values ("More Value per Key" §5.2).
    Caches are [B, h, max_seq_len, width] bf16 (h = h_k for keys, h_v for
    values); ``seq_lens`` int32 [B] gives the valid positions of each row.
    """

    def __init__(self, max_batch: int, max_seq_len: int, h_q: int, h_k: int, h_v: int,
                 head_dim: int, max_N: int, device=None, head_dim_v=None):
        self.lib = load()
        self.max_batch, self.max_seq_len = max_batch, max_seq_len
        self.h_q, self.h_k, self.h_v, self.head_dim, self.max_N = h_q, h_k, h_v, head_dim, max_N
        self.head_dim_v = head_dim if head_dim_v is None else head_dim_v
        self.batch = max_batch
        if device is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        else:
            dev = torch.device(device)
            self.device = torch.device("cuda", dev.index if dev.index is not None else 0)
        self._h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            stream = torch.cuda.current_stream(self.device).cuda_stream
            _lib.check("saga_decode_init_kv", self.lib.saga_decode_init_kv(
                ctypes.byref(self._h), max_batch, max_seq_len, h_q, h_k, h_v, head_dim,
                self.head_dim_v, max_N, ctypes.c_void_p(stream)))

    # ------------------------------------------------------------------ plumbing
    def _stream(self):
        s = torch.cuda.current_stream(self.device).cuda_stream
        _lib.check("saga_decode_set_stream", self.lib.saga_decode_set_stream(self._h, ctypes.c_void_p(s)))

    def set_batch(self, batch: int):
        _lib.check("saga_decode_set_batch", self.lib.saga_decode_set_batch(self._h, batch))
        self.batch = batch

    def _check_caches(self, q, k_cache, v_cache, seq_lens):
        B, L, d = self.batch, self.max_seq_len, self.head_dim
        if q is not None:
            _need(q, "q", torch.bfloat16, (B, self.h_q, d), "cuda")
        if k_cache is not None:
            _need(k_cache, "k_cache", torch.bfloat16, (B, self.h_k, L, d), "cuda")
        if v_cache is not None:
            _need(v_cache, "v_cache", torch.bfloat16, (B, self.h_v, L, self.head_dim_v), "cuda")
        if seq_lens is not None:
            _need(seq_lens, "seq_lens", torch.int32, (B,), "cuda")

    # ------------------------------------------------------------------ calls
    def attn(self, q, k_cache, v_cache, seq_lens, N: int, out=None, sel_idx=None, sel_logit=None):
        """Decode step: out[b, j] = softmax(z[I]) V[I] over the top-N positions I."""
        self._check_caches(q, k_cache, v_cache, seq_lens)
        B = self.batch
        if out is None:
            out = torch.empty(B, self.h_q, self.head_dim_v, dtype=torch.bfloat16, device=q.device)
        _need(out, "out", torch.bfloat16, (B, self.h_q, self.head_dim_v), "cuda")
        if sel_idx is not None:
            _need(sel_idx, "sel_idx", torch.int32, (B, self.h_q, N), "cuda")
        if sel_logit is not None:
            _need(sel_logit, "sel_logit", torch.float32, (B, self.h_q, N), "cuda")
        self._stream()
        args = (self._h, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                self.h_q, self.h_k, self.h_v, self.head_dim, N, _ptr(out))
        if sel_idx is None and sel_logit is None:
            _lib.check("saga_decode_attn", self.lib.saga_decode_attn(*args))
        else:
            _lib.check("saga_decode_attn_ex",
                       self.lib.saga_decode_attn_ex(*args, _ptr(sel_idx), _ptr(sel_logit)))
        return out

    def group_attn(self, q, k_cache, v_cache, seq_lens, N: int, out=None, sel_idx=None,
                   sel_stat=None, sel_logit=None):
        """Group-shared selection: one set of N positions per value head (the largest
        summed softmax probabilities of its query heads), each head's own softmax over
        it and the gathered P.V.  sel_idx / sel_stat [B, h_v, N], sel_logit [B, h_q, N]."""
        self._check_caches(q, k_cache, v_cache, seq_lens)
        B = self.batch
        if out is None:
            out = torch.empty(B, self.h_q, self.head_dim_v, dtype=torch.bfloat16, device=q.device)
        _need(out, "out", torch.bfloat16, (B, self.h_q, self.head_dim_v), "cuda")
        if sel_idx is not None:
            _need(sel_idx, "sel_idx", torch.int32, (B, self.h_v, N), "cuda")
        if sel_stat is not None:
            _need(sel_stat, "sel_stat", torch.float32, (B, self.h_v, N), "cuda")
        if sel_logit is not None:
            _need(sel_logit, "sel_logit", torch.float32, (B, self.h_q, N), "cuda")
        self._stream()
        _lib.check("saga_group_attn", self.lib.saga_group_attn(
            self._h, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), self.h_q, self.h_k,
            self.h_v, self.head_dim, N, _ptr(out), _ptr(sel_idx), _ptr(sel_stat), _ptr(sel_logit)))
        return out

    def atopn_calibrate(self, q, k_cache, v_cache, seq_lens, N: int, log_tau=None, out=None,
                        sel_idx=None, sel_logit=None):
        """Calibration step of stateful Atop-N: the exact top-N decode step, and per row
        log tau = log of the softmax probability of the N-th largest score.

        Returns (out, log_tau); log_tau is fp32 [B, h_q], the state that later
        ``atopn_step`` calls reuse.
        """
        self._check_caches(q, k_cache, v_cache, seq_lens)
        B = self.batch
        if out is None:
            out = torch.empty(B, self.h_q, self.head_dim_v, dtype=torch.bfloat16, device=q.device)
        if log_tau is None:
            log_tau = torch.empty(B, self.h_q, dtype=torch.float32, device=q.device)
        _need(out, "out", torch.bfloat16, (B, self.h_q, self.head_dim_v), "cuda")
        _need(log_tau, "log_tau", torch.float32, (B, self.h_q), "cuda")
        if sel_idx is not None:
            _need(sel_idx, "sel_idx", torch.int32, (B, self.h_q, N), "cuda")
        if sel_logit is not None:
            _need(sel_logit, "sel_logit", torch.float32, (B, self.h_q, N), "cuda")
        self._stream()
        _lib.check("saga_atopn_calibrate", self.lib.saga_atopn_calibrate(
            self._h, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), self.h_q, self.h_k,
            self.h_v, self.head_dim, N, _ptr(out), _ptr(sel_idx), _ptr(sel_logit), _ptr(log_tau)))
        return out, log_tau

    def atopn_step(self, q, k_cache, v_cache, seq_lens, N: int, log_tau, out=None,
                   sel_idx=None, sel_logit=None):
        """A step of stateful Atop-N: keep every score z >= log_tau + logsumexp(z) (the
        first 2N positions), softmax over them and the gathered P.V.

        sel_idx / sel_logit, if given, are [B, h_q, 2N] (padding -1 / -inf).
        """
        self._check_caches(q, k_cache, v_cache, seq_lens)
        B = self.batch
        if out is None:
            out = torch.empty(B, self.h_q, self.head_dim_v, dtype=torch.bfloat16, device=q.device)
        _need(out, "out", torch.bfloat16, (B, self.h_q, self.head_dim_v), "cuda")
        _need(log_tau, "log_tau", torch.float32, (B, self.h_q), "cuda")
        if sel_idx is not None:
            _need(sel_idx, "sel_idx", torch.int32, (B, self.h_q, 2 * N), "cuda")
        if sel_logit is not None:
            _need(sel_logit, "sel_logit", torch.float32, (B, self.h_q, 2 * N), "cuda")
        self._stream()
        _lib.check("saga_atopn_step", self.lib.saga_atopn_step(
            self._h, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), self.h_q, self.h_k,
            self.h_v, self.head_dim, N, _ptr(log_tau), _ptr(out), _ptr(sel_idx), _ptr(sel_logit)))
        return out

    def attn_host(self, q_host, k_cache, v_cache, seq_lens_host, N: int, out_host):
        """Decode step with q / seq_lens / out in (pinned) host memory; asynchronous."""
        B = self.batch
        _need(q_host, "q_host", torch.bfloat16, (B, self.h_q, self.head_dim), "cpu")
        _need(seq_lens_host, "seq_lens_host", torch.int32, (B,), "cpu")
        _need(out_host, "out_host", torch.bfloat16, (B, self.h_q, self.head_dim_v), "cpu")
        self._check_caches(None, k_cache, v_cache, None)
        self._stream()
        _lib.check("saga_decode_attn_host", self.lib.saga_decode_attn_host(
            self._h, _ptr(q_host), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens_host),
            self.h_q, self.h_k, self.h_v, self.head_dim, N, _ptr(out_host)))
        return out_host

    def score(self, q, k_cache, seq_lens, scores=None):
        """Stage S1: fp32 scores [B, h_q, max_seq_len] (positions >= L_b not written)."""
        self._check_caches(q, k_cache, None, seq_lens)
        if scores is None:
            scores = torch.full((self.batch, self.h_q, self.max_seq_len), float("nan"),
                                dtype=torch.float32, device=q.device)
        _need(scores, "scores", torch.float32, device="cuda")
        if scores.dim() != 3 or scores.shape[:2] != (self.batch, self.h_q):
            raise ValueError("scores must be [B, h_q, stride]")
        self._stream()
        _lib.check("saga_score", self.lib.saga_score(
            self._h, _ptr(q), _ptr(k_cache), _ptr(seq_lens), self.h_q, self.h_k, self.head_dim,
            _ptr(scores), scores.shape[2]))
        return scores

    def select(self, scores, seq_lens, N: int, sel_idx=None, sel_logit=None):
        """Stage S2: exact top-N of each fp32 score row, ties to the lowest index."""
        B = self.batch
        _need(scores, "scores", torch.float32, device="cuda")
        _need(seq_lens, "seq_lens", torch.int32, (B,), "cuda")
        if sel_idx is None:
            sel_idx = torch.empty(B, self.h_q, N, dtype=torch.int32, device=scores.device)
        if sel_logit is None:
            sel_logit = torch.empty(B, self.h_q, N, dtype=torch.float32, device=scores.device)
        _need(sel_idx, "sel_idx", torch.int32, (B, self.h_q, N), "cuda")
        _need(sel_logit, "sel_logit", torch.float32, (B, self.h_q, N), "cuda")
        self._stream()
        _lib.check("saga_select", self.lib.saga_select(
            self._h, _ptr(scores), scores.shape[2], _ptr(seq_lens), self.h_q, N,
            _ptr(sel_idx), _ptr(sel_logit)))
        return sel_idx, sel_logit

    def combine(self, sel_idx, sel_logit, v_cache, seq_lens, out=None):
        """Stages S3 + S4: softmax over a selection and the gathered P.V."""
        B = self.batch
        N = sel_idx.shape[-1]
        _need(sel_idx, "sel_idx", torch.int32, (B, self.h_q, N), "cuda")
        _need(sel_logit, "sel_logit", torch.float32, (B, self.h_q, N), "cuda")
        self._check_caches(None, None, v_cache, seq_lens)
        if out is None:
            out = torch.empty(B, self.h_q, self.head_dim_v, dtype=torch.bfloat16, device=v_cache.device)
        _need(out, "out", torch.bfloat16, (B, self.h_q, self.head_dim_v), "cuda")
        self._stream()
        _lib.check("saga_combine", self.lib.saga_combine(
            self._h, _ptr(sel_idx), _ptr(sel_logit), _ptr(v_cache), _ptr(seq_lens),
            self.h_q, self.h_v, self.head_dim_v, N, _ptr(out)))
        return out

    # ------------------------------------------------------------------ status
    def status(self) -> int:
        """Synchronise; return and clear the device status word (no exception)."""
        self._stream()
        v = ctypes.c_int(0)
        rc = self.lib.saga_decode_status(self._h, ctypes.byref(v))
        if rc not in (_lib.SAGA_OK, _lib.SAGA_ERR_DEVICE):
            raise SagaError("saga_decode_status", rc)
        return v.value

    def selftest_timeout(self):
        """Failure-detection self-test: a kernel whose bounded wait runs out sets
        SAGA_STATUS_TIMEOUT (read it with ``status()``); asynchronous, ~2 s."""
        self._stream()
        _lib.check("saga_decode_selftest_timeout", self.lib.saga_decode_selftest_timeout(self._h))

    def launch_count(self) -> int:
        v = ctypes.c_longlong(0)
        _lib.check("saga_decode_launch_count", self.lib.saga_decode_launch_count(self._h, ctypes.byref(v)))
        return v.value

    def profile(self, enable: bool, max_calls: int = 0):
        _lib.check("saga_decode_profile", self.lib.saga_decode_profile(self._h, int(enable), max_calls))

    def profile_read(self):
        s, c, n = ctypes.c_double(), ctypes.c_double(), ctypes.c_int()
        _lib.check("saga_decode_profile_read", self.lib.saga_decode_profile_read(
            self._h, ctypes.byref(s), ctypes.byref(c), ctypes.byref(n)))
        return s.value, c.value, n.value

    def close(self):
        if self._h:
            rc = self.lib.saga_decode_free(self._h)
            self._h = ctypes.c_void_p()
            _lib.check("saga_decode_free", rc)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def combine_noalloc(sel_idx, sel_logit, v_cache, seq_lens, out):
    """Softmax over a selection and the gathered P.V (stages S3 + S4) without a handle.

    For callers that cannot allocate device memory -- e.g. a serving engine whose memory
    manager owns the whole device, or a process under a hard memory cap -- and so cannot
    create a SagaDecoder (its workspace is allocated).  This function allocates nothing, not
    even the output: ``out`` (bf16 [B, h_q, d]) must be supplied.  The library keeps the
    kernel's scratch in a fixed 4 MiB array of its own; problems that do not fit raise
    SagaError (SAGA_ERR_SCRATCH_TOO_SMALL).  The first call on a device should come before
    any stream capture, and calls on different streams must not overlap on the GPU.
    sel_idx / sel_logit: [B, h_q, N] (index -1 = padding); v_cache: [B, h_v, L_max, d] bf16;
    seq_lens: [B] int32, all on out's device.  Runs on that device's current stream,
    asynchronously.  Data errors only the device sees are not reported (there is no handle
    and so no status word): a row whose seq_len lies outside [1, L_max] gets zeros and an
    index >= its row's seq_len is skipped.
    """
    lib = load()
    B, h_q, N = sel_idx.shape
    _need(sel_idx, "sel_idx", torch.int32, (B, h_q, N), "cuda")
    _need(sel_logit, "sel_logit", torch.float32, (B, h_q, N), "cuda")
    _need(v_cache, "v_cache", torch.bfloat16, device="cuda")
    if v_cache.dim() != 4 or v_cache.shape[0] != B:
        raise ValueError("v_cache must be [B, h_v, L_max, d]")
    _, h_v, L_max, d = v_cache.shape
    _need(seq_lens, "seq_lens", torch.int32, (B,), "cuda")
    _need(out, "out", torch.bfloat16, (B, h_q, d), "cuda")
    for name, t in (("sel_idx", sel_idx), ("sel_logit", sel_logit), ("v_cache", v_cache),
                    ("seq_lens", seq_lens)):
        if t.device != out.device:
            raise ValueError(f"{name} is on {t.device}, out on {out.device}: one device for all")
    # the library looks up its scratch on the current device and runs on its current stream
    with torch.cuda.device(out.device):
        stream = torch.cuda.current_stream(out.device).cuda_stream
        _lib.check("saga_combine_noalloc", lib.saga_combine_noalloc(
            _ptr(sel_idx), _ptr(sel_logit), _ptr(v_cache), _ptr(seq_lens), B, L_max, h_q, h_v, d,
            N, _ptr(out), ctypes.c_void_p(stream)))
    return out
