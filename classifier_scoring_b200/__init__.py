"""Python binding of librmscore, the B200 transformer scorer (C ABI in include/rm.h).

Argument marshalling only: every step of the scoring path runs in the CUDA
library.  Device buffers are passed as objects with ``data_ptr()`` (torch
tensors) or raw integer addresses; streams as objects with ``cuda_stream``
(torch streams), integers, or None for the default stream.  If the library
is not built this module raises on first use; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import weakref
from typing import Optional

import numpy as np

__all__ = ["RmConfig", "RmError", "Scorer", "lib", "schedule", "weights_bytes", "ops",
           "ENC_POSTLN", "DEC_PRELN", "F32", "BF16", "GELU_ERF", "GELU_TANH"]

ENC_POSTLN, DEC_PRELN = 0, 1
F32, BF16 = 0, 1
ROWS_RESID_F32 = 2          # res_ln rows: x fp32, y and z bf16
ROWS_F32_IN = 3             # res_ln rows: y and x fp32, z bf16
GELU_ERF, GELU_TANH = 0, 1
ATTN_FUSED, ATTN_MATERIALIZED = 0, 1
RM_OK, RM_E_INVAL, RM_E_NOMEM, RM_E_CUDA, RM_E_RANGE, RM_E_DEVICE = 0, -1, -2, -3, -4, -5
SCHED_THROUGHPUT, SCHED_LATENCY = 0, 1

# RMSCORE_LIB names another build of the library (the checked build,
# librmscore_checked.so, for tests of its bounds checks)
LIB_PATH = os.environ.get("RMSCORE_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                         "librmscore.so")
CHECKED_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librmscore_checked.so")


class RmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"rm error {code}: {msg}")
        self.code = code


class RmConfig(ctypes.Structure):
    _fields_ = [
        ("arch", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32),
        ("n_heads", ctypes.c_int32), ("ffn", ctypes.c_int32), ("vocab", ctypes.c_int32),
        ("max_pos", ctypes.c_int32), ("weight_dtype", ctypes.c_int32), ("gelu", ctypes.c_int32),
        ("ln_eps", ctypes.c_float),
        ("max_batch_seqs", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("max_len", ctypes.c_int32),
        ("sched_max_batch", ctypes.c_int32), ("sched_c0", ctypes.c_int64), ("sched_c1", ctypes.c_int64),
        ("sched_table", ctypes.POINTER(ctypes.c_int64)), ("sched_table_b", ctypes.c_int32),
        ("sched_table_l", ctypes.c_int32), ("attn_impl", ctypes.c_int32),
        ("sched_objective", ctypes.c_int32), ("sched_max_cost", ctypes.c_int64),
    ]

    @classmethod
    def make(cls, *, arch, n_layers, hidden, n_heads, ffn, vocab, max_pos, weight_dtype,
             gelu=GELU_ERF, ln_eps=1e-12, max_batch_seqs=64, max_tokens=8192, max_len=512,
             sched_max_batch=64, sched_c0=0, sched_c1=1, sched_table=None,
             attn_impl=0, sched_objective=0, sched_max_cost=0) -> "RmConfig":
        c = cls(arch, n_layers, hidden, n_heads, ffn, vocab, max_pos, weight_dtype, gelu, ln_eps,
                max_batch_seqs, max_tokens, max_len, sched_max_batch, sched_c0, sched_c1, None, 0, 0,
                attn_impl, sched_objective, sched_max_cost)
        if sched_table is not None:
            t = np.ascontiguousarray(sched_table, dtype=np.int64)
            c._table_keepalive = t
            c.sched_table = t.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
            c.sched_table_b, c.sched_table_l = int(t.shape[0]), int(t.shape[1])
        return c


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m classifier_scoring_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    cfgp = ctypes.POINTER(RmConfig)
    sig = {
        "rm_weights_bytes": (SZ, [cfgp]),
        "rm_create": (ctypes.c_int, [cfgp, P, SZ, ctypes.POINTER(P)]),
        "rm_create_shared": (ctypes.c_int, [P, ctypes.POINTER(P)]),
        "rm_score": (ctypes.c_int, [P, P, P, I32, P, P]),
        "rm_score_prefix": (ctypes.c_int, [P, P, P, P, P, I32, P, P, P, P]),
        "rm_plan_create": (ctypes.c_int, [P, P, I32, P]),
        "rm_score_plan": (ctypes.c_int, [P, P, P, P]),
        "rm_plan_destroy": (None, [P]),
        "rm_score_host": (ctypes.c_int, [P, P, P, I32, P, P]),
        "rm_schedule": (ctypes.c_int, [P, P, I32, P]),
        "rm_schedule_cfg": (ctypes.c_int, [cfgp, P, I32, P]),
        "rm_get_device_error": (ctypes.c_int, [P, P]),
        "rm_arena_stats": (ctypes.c_int, [P, P]),
        "rm_selftest_bounded_wait": (ctypes.c_int, [I64, P, P]),
        "rm_debug_fail_alloc": (ctypes.c_int, [I32]),
        "rm_build_checked": (ctypes.c_int, []),
        "rm_bounds_errors": (ctypes.c_int, [P]),
        "rm_destroy": (None, [P]),
        "rm_profile": (ctypes.c_int, [P, I32]),
        "rm_profile_read": (ctypes.c_int, [P, P, P, P, P, P]),
        "rm_last_error": (ctypes.c_char_p, []),
        "rm_varlen_meta": (ctypes.c_int, [P, I32, I32, P, P]),
        "rm_op_gemm": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I32, I32, P]),
        "rm_op_gemm_tiled": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I32, I32, I32, I32, P]),
        "rm_op_gemm_accumulate": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I32, I32, I32, I32, P]),
        "rm_gemm_tile": (ctypes.c_int, [I32, I32, I32, I32, P]),
        "rm_op_vote": (ctypes.c_int, [P, I32, I32, F, P, P, P]),
        "rm_op_embed": (ctypes.c_int, [P, P, I32, I32, P, P, P, P, F, I32, I32, I32, P, I32, P, P]),
        "rm_op_attn_scores": (ctypes.c_int, [P, P, P, P, P, I32, I32, I32, I32, I32, P]),
        "rm_op_softmax": (ctypes.c_int, [P, I32, P, P, I32, I32, I32, I32, I32, P]),
        "rm_op_softmax_classes": (ctypes.c_int, [P, I32, P, P, I32, I32, I32, I32, I32, P, P]),
        "rm_softmax_scratch_bytes": (SZ, [I32, I32, I32]),
        "rm_op_attn_context": (ctypes.c_int, [P, P, P, P, P, P, I32, I32, I32, I32, I32, P]),
        "rm_op_attn_fused": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I32, I32, P]),
        "rm_op_attention_noalloc": (ctypes.c_int, [P, P, P, I32, I32, I32, I32, P]),
        "rm_op_attn_tiles": (ctypes.c_int, [P, P, P, I32, I32, I32, I32, I32, I32, P]),
        "rm_attn_tc_tiles": (ctypes.c_int, [P, I32, P]),
        "rm_op_attn_tc": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I32, I32, P]),
        "rm_attn_tcl_items": (ctypes.c_int, [P, I32, I32, P]),
        "rm_op_attn_tcl": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I32, I32, P]),
        "rm_op_res_ln": (ctypes.c_int, [P, P, P, P, P, I32, I32, F, I32, I32, P]),
        "rm_op_head": (ctypes.c_int, [P, P, I32, P, F, I32, I32, P, P]),
        "rm_arena_plan": (ctypes.c_int, [cfgp, I32, I32, I64, P, P, P, P, I32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(rc: int) -> int:
    if rc < 0:
        raise RmError(rc, lib().rm_last_error().decode())
    return rc


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return int(x)


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    return int(s)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def weights_bytes(cfg: RmConfig) -> int:
    return lib().rm_weights_bytes(ctypes.byref(cfg))


def schedule(cfg: RmConfig, lengths) -> np.ndarray:
    """DP batch assignment of a request queue (host only, rm_schedule_cfg)."""
    ln = _i32(lengths)
    out = np.empty(len(ln), dtype=np.int32)
    _check(lib().rm_schedule_cfg(ctypes.byref(cfg), ln.ctypes.data, len(ln), out.ctypes.data))
    return out


class Scorer:
    """A scorer handle (rm_create ... rm_destroy)."""

    def __init__(self, cfg: RmConfig, weights: np.ndarray = None, *, share: "Scorer" = None):
        h = ctypes.c_void_p()
        if share is not None:
            _check(lib().rm_create_shared(share._h, ctypes.byref(h)))
            cfg = share.cfg
        else:
            w = np.ascontiguousarray(weights)
            _check(lib().rm_create(ctypes.byref(cfg), w.ctypes.data, w.nbytes, ctypes.byref(h)))
        self._h = h
        self.cfg = cfg
        self._plans = weakref.WeakSet()          # plans on this handle, closed with it

    def shared(self) -> "Scorer":
        """A new handle on the same weights with its own arena (rm_create_shared)."""
        return Scorer(self.cfg, share=self)

    def close(self):
        # a plan uses its handle's arena: plans go first (rm_plan_destroy before rm_destroy)
        for p in list(getattr(self, "_plans", ())):
            p.close()
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().rm_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    def score(self, ids_dev, offsets, out_dev, stream=None) -> None:
        """rm_score: device ids/out, host offsets (int32[n+1])."""
        off = _i32(offsets)
        _check(lib().rm_score(self._h, _ptr(ids_dev), off.ctypes.data, len(off) - 1, _ptr(out_dev),
                              _stream(stream)))

    def score_prefix(self, ids_dev, prefix_len, n_cand, cand_len, out_dev, best_dev=None,
                     logodds_dev=None, stream=None) -> None:
        """rm_score_prefix: candidates sharing a prefix; host group layout, device ids/outputs."""
        pl, nc, cl = _i32(prefix_len), _i32(n_cand), _i32(cand_len)
        _check(lib().rm_score_prefix(self._h, _ptr(ids_dev), pl.ctypes.data, nc.ctypes.data,
                                     cl.ctypes.data, len(pl), _ptr(out_dev), _ptr(best_dev),
                                     _ptr(logodds_dev), _stream(stream)))

    def plan(self, offsets) -> "Plan":
        """rm_plan_create: a prepared batch shape for launch-only scoring."""
        p = Plan(self, offsets)
        self._plans.add(p)
        return p

    def score_host(self, ids_host, offsets, out_host, stream=None) -> None:
        """rm_score_host: host ids/out (pinned for asynchronous copies)."""
        off = _i32(offsets)
        _check(lib().rm_score_host(self._h, _ptr(ids_host), off.ctypes.data, len(off) - 1,
                                   _ptr(out_host), _stream(stream)))

    def schedule(self, lengths) -> np.ndarray:
        ln = _i32(lengths)
        out = np.empty(len(ln), dtype=np.int32)
        _check(lib().rm_schedule(self._h, ln.ctypes.data, len(ln), out.ctypes.data))
        return out

    def device_error(self) -> np.ndarray:
        out = np.zeros(2, dtype=np.int32)
        _check(lib().rm_get_device_error(self._h, out.ctypes.data))
        return out

    K_NAMES = ("gemm", "attn_scores", "softmax", "attn_context", "layernorm", "embed", "head",
               "attn_fused")

    def profile(self, every: int) -> None:
        """Time every-th call's launches with CUDA events (0 = off); restarts counters."""
        _check(lib().rm_profile(self._h, int(every)))

    def profile_read(self) -> dict:
        """Per kernel class: ms, launches, flops, bytes of the timed launches; plus total launches."""
        k = len(self.K_NAMES)
        ms, nl = np.zeros(k), np.zeros(k, dtype=np.int64)
        fl, by = np.zeros(k), np.zeros(k)
        tot = np.zeros(1, dtype=np.int64)
        _check(lib().rm_profile_read(self._h, ms.ctypes.data, nl.ctypes.data, fl.ctypes.data,
                                     by.ctypes.data, tot.ctypes.data))
        out = {name: {"ms": float(ms[i]), "launches": int(nl[i]), "flops": float(fl[i]),
                      "bytes": float(by[i])} for i, name in enumerate(self.K_NAMES)}
        out["total_launches"] = int(tot[0])
        return out

    def arena_stats(self) -> np.ndarray:
        out = np.zeros(3, dtype=np.int64)
        _check(lib().rm_arena_stats(self._h, out.ctypes.data))
        return out


class ops:
    """Per-step entry points of include/rm_ops.h (device pointers)."""

    @staticmethod
    def varlen_meta(offsets, n_heads):
        off = _i32(offsets)
        n = len(off) - 1
        rb = np.zeros(n + 1, dtype=np.int32)
        so = np.zeros(n + 1, dtype=np.int64)
        _check(lib().rm_varlen_meta(off.ctypes.data, n, n_heads, rb.ctypes.data, so.ctypes.data))
        return rb, so

    @staticmethod
    def gemm(x, w, bias, y, y_dtype, M, N, K, act=0, stream=None):
        _check(lib().rm_op_gemm(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), y_dtype, M, N, K, act,
                                _stream(stream)))

    @staticmethod
    def gemm_tiled(x, w, bias, y, y_dtype, M, N, K, act=0, cg=0, bn=0, stream=None):
        _check(lib().rm_op_gemm_tiled(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), y_dtype, M, N, K,
                                      act, cg, bn, _stream(stream)))

    @staticmethod
    def gemm_accumulate(x, w, bias, y, y_dtype, M, N, K, act=0, cg=0, bn=0, stream=None):
        _check(lib().rm_op_gemm_accumulate(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), y_dtype, M, N,
                                           K, act, cg, bn, _stream(stream)))

    @staticmethod
    def vote(scores, K, n, threshold=0.0, decision=None, votes=None, stream=None):
        _check(lib().rm_op_vote(_ptr(scores), K, n, threshold, _ptr(decision), _ptr(votes),
                                _stream(stream)))

    @staticmethod
    def gemm_tile(M, N, K, num_sms):
        out = np.zeros(2, dtype=np.int32)
        _check(lib().rm_gemm_tile(M, N, K, num_sms, out.ctypes.data))
        return int(out[0]), int(out[1])

    @staticmethod
    def embed(ids, offsets_dev, n_seqs, T, emb_word, emb_pos, ln_g, ln_b, eps, V, P, H, x,
              err_count=None, stream=None, x_dtype=BF16):
        _check(lib().rm_op_embed(_ptr(ids), _ptr(offsets_dev), n_seqs, T, _ptr(emb_word),
                                 _ptr(emb_pos), _ptr(ln_g), _ptr(ln_b), eps, V, P, H, _ptr(x),
                                 x_dtype, _ptr(err_count), _stream(stream)))

    @staticmethod
    def attn_scores(qkv, S, offsets_dev, rb_dev, so_dev, n_seqs, n_row_blocks, n_heads, head_dim,
                    causal, stream=None):
        _check(lib().rm_op_attn_scores(_ptr(qkv), _ptr(S), _ptr(offsets_dev), _ptr(rb_dev),
                                       _ptr(so_dev), n_seqs, n_row_blocks, n_heads, head_dim,
                                       int(causal), _stream(stream)))

    @staticmethod
    def softmax(S, s_dtype, offsets_dev, so_dev, n_seqs, T, n_heads, max_len, causal, stream=None):
        _check(lib().rm_op_softmax(_ptr(S), s_dtype, _ptr(offsets_dev), _ptr(so_dev), n_seqs, T,
                                   n_heads, max_len, int(causal), _stream(stream)))

    @staticmethod
    def softmax_scratch_bytes(n_seqs, T, n_heads):
        return int(lib().rm_softmax_scratch_bytes(int(n_seqs), int(T), int(n_heads)))

    @staticmethod
    def softmax_classes(S, s_dtype, offsets_dev, so_dev, n_seqs, T, n_heads, max_len, causal, scratch,
                        stream=None):
        """scratch: device buffer of softmax_scratch_bytes(n_seqs, T, n_heads) bytes."""
        _check(lib().rm_op_softmax_classes(_ptr(S), s_dtype, _ptr(offsets_dev), _ptr(so_dev), n_seqs,
                                           T, n_heads, max_len, causal, _ptr(scratch), _stream(stream)))

    @staticmethod
    def attn_context(S, qkv, ctx, offsets_dev, rb_dev, so_dev, n_seqs, n_row_blocks, n_heads,
                     head_dim, causal, stream=None):
        _check(lib().rm_op_attn_context(_ptr(S), _ptr(qkv), _ptr(ctx), _ptr(offsets_dev),
                                        _ptr(rb_dev), _ptr(so_dev), n_seqs, n_row_blocks, n_heads,
                                        head_dim, int(causal), _stream(stream)))

    @staticmethod
    def attn_fused(qkv, ctx, offsets_dev, rb_dev, n_seqs, n_row_blocks, n_heads, head_dim, causal,
                   stream=None):
        _check(lib().rm_op_attn_fused(_ptr(qkv), _ptr(ctx), _ptr(offsets_dev), _ptr(rb_dev), n_seqs,
                                      n_row_blocks, n_heads, head_dim, int(causal), _stream(stream)))

    @staticmethod
    def attn_tiles(qkv, ctx, offsets_dev, n_seqs, T, n_heads, head_dim, causal, stream=None,
                   max_len=None):
        """max_len: bound on the sequence lengths (default T)."""
        _check(lib().rm_op_attn_tiles(_ptr(qkv), _ptr(ctx), _ptr(offsets_dev), n_seqs, T, n_heads,
                                      head_dim, T if max_len is None else max_len, causal,
                                      _stream(stream)))

    @staticmethod
    def attn_tc_tiles(offsets):
        """rm_attn_tc_tiles: host offsets -> int32 tile boundaries (sequence indices)."""
        off = _i32(offsets)
        n = len(off) - 1
        out = np.zeros(n + 1, dtype=np.int32)
        k = _check(lib().rm_attn_tc_tiles(off.ctypes.data, n, out.ctypes.data))
        return out[:k + 1].copy()

    @staticmethod
    def attn_tcl_items(offsets, causal=0):
        """rm_attn_tcl_items: host offsets -> int32 work items of the long-row kernel."""
        off = _i32(offsets)
        n = len(off) - 1
        out = np.zeros(4 * n, dtype=np.int32)
        k = _check(lib().rm_attn_tcl_items(off.ctypes.data, n, causal, out.ctypes.data))
        return out[:k].copy()

    @staticmethod
    def attn_tcl(qkv, ctx, offsets_dev, items_dev, n_items, n_seqs, T, n_heads, causal, stream=None):
        _check(lib().rm_op_attn_tcl(_ptr(qkv), _ptr(ctx), _ptr(offsets_dev), _ptr(items_dev), n_items,
                                    n_seqs, T, n_heads, causal, _stream(stream)))

    @staticmethod
    def attn_tc(qkv, ctx, offsets_dev, tiles_dev, n_tiles, n_seqs, T, n_heads, causal, stream=None):
        _check(lib().rm_op_attn_tc(_ptr(qkv), _ptr(ctx), _ptr(offsets_dev), _ptr(tiles_dev), n_tiles,
                                   n_seqs, T, n_heads, causal, _stream(stream)))

    @staticmethod
    def attention_noalloc(qkv, ctx, offsets, n_heads, head_dim, causal, stream=None):
        """rm_op_attention_noalloc: host offsets; scratch in the library's static array."""
        off = _i32(offsets)
        _check(lib().rm_op_attention_noalloc(_ptr(qkv), _ptr(ctx), off.ctypes.data, len(off) - 1,
                                             n_heads, head_dim, int(causal), _stream(stream)))

    @staticmethod
    def res_ln(y, x, z, g, b, T, H, eps, dtype, mode, stream=None):
        _check(lib().rm_op_res_ln(_ptr(y), _ptr(x), _ptr(z), _ptr(g), _ptr(b), T, H, eps, dtype,
                                  mode, _stream(stream)))

    @staticmethod
    def head(x, offsets_dev, n_seqs, w_r, b_r, H, last_token, out, stream=None):
        _check(lib().rm_op_head(_ptr(x), _ptr(offsets_dev), n_seqs, _ptr(w_r), b_r, H,
                                int(last_token), _ptr(out), _stream(stream)))

    @staticmethod
    def arena_plan(cfg: RmConfig, T, n_seqs, s_elems, max_bufs=16):
        off = np.zeros(max_bufs, dtype=np.int64)
        nb = np.zeros(max_bufs, dtype=np.int64)
        first = np.zeros(max_bufs, dtype=np.int32)
        last = np.zeros(max_bufs, dtype=np.int32)
        peak = np.zeros(1, dtype=np.int64)
        k = _check(lib().rm_arena_plan(ctypes.byref(cfg), T, n_seqs, s_elems, off.ctypes.data,
                                       nb.ctypes.data, first.ctypes.data, last.ctypes.data,
                                       max_bufs, peak.ctypes.data))
        return off[:k], nb[:k], first[:k], last[:k], int(peak[0])


class Plan:
    """rm_plan: the batch shape of repeated calls, prepared once; score() only
    enqueues kernels (capturable in a CUDA graph)."""

    def __init__(self, scorer: "Scorer", offsets):
        self._scorer = scorer                  # keeps the handle alive
        off = _i32(offsets)
        h = ctypes.c_void_p()
        _check(lib().rm_plan_create(scorer._h, off.ctypes.data, len(off) - 1, ctypes.byref(h)))
        self._p = h
        self.n = len(off) - 1

    def score(self, ids_dev, out_dev, stream=None) -> None:
        if not self._p:
            raise RmError(RM_E_INVAL, "the plan (or its scorer) has been closed")
        _check(lib().rm_score_plan(self._p, _ptr(ids_dev), _ptr(out_dev), _stream(stream)))

    def close(self):
        if self._p:
            lib().rm_plan_destroy(self._p)
            self._p = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def build_checked() -> bool:
    """True in the checked build (librmscore_checked.so)."""
    return bool(lib().rm_build_checked())


def bounds_errors() -> int:
    """rm_bounds_errors: failed bounds tests since the last call (checked build)."""
    out = np.zeros(1, dtype=np.int64)
    _check(lib().rm_bounds_errors(out.ctypes.data))
    return int(out[0])


def debug_fail_alloc(k: int) -> None:
    """rm_debug_fail_alloc: the k-th library allocation from now on fails (0 disarms)."""
    _check(lib().rm_debug_fail_alloc(int(k)))


def selftest_bounded_wait(limit_ns: int):
    """rm_selftest_bounded_wait: (timed_out, elapsed_ns) of a wait that nothing ends."""
    flag = ctypes.c_int32()
    ns = ctypes.c_int64()
    _check(lib().rm_selftest_bounded_wait(int(limit_ns), ctypes.byref(flag), ctypes.byref(ns)))
    return int(flag.value), int(ns.value)
