"""ctypes binding of libduolm.so: argument marshalling only.

Each ``Ranker`` method calls the C entry point of the same name
(``duolm_<name>``); arrays are checked for dtype and contiguity and passed as
pointers.  No step of the ranker runs in Python.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libduolm.so")

DTYPE_FP32 = 0
DTYPE_BF16 = 1
MODE_MIS = 0
MODE_INDEPENDENT = 1

_ERRORS = {-1: "DUOLM_E_ARG", -2: "DUOLM_E_ID", -3: "DUOLM_E_OFFSETS", -4: "DUOLM_E_EMPTY",
           -5: "DUOLM_E_CAPACITY", -6: "DUOLM_E_CUDA", -7: "DUOLM_E_DEVICE", -8: "DUOLM_E_STATE"}


class DuolmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_ERRORS.get(code, code)}: {msg}")
        self.code = code


class ModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("dtype", ctypes.c_int)]


class Template(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int32), ("marker", ctypes.c_int32), ("m", ctypes.c_int32),
                ("instr", ctypes.c_void_p), ("n_instr", ctypes.c_int32),
                ("header", ctypes.c_void_p), ("n_header", ctypes.c_int32),
                ("branch_header", ctypes.c_void_p), ("n_branch_header", ctypes.c_int32)]


def _load():
    if not os.path.exists(lib_path):
        raise ImportError(f"{lib_path} is missing: build it with `python -m shared_prefix_item_b200.build`")
    L = ctypes.CDLL(lib_path)
    P, I, I64, VP = ctypes.POINTER, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
    sig = {
        "duolm_weight_count": (I, [P(ModelDesc)]),
        "duolm_model_load": (I, [P(ModelDesc), VP, I, VP, P(VP)]),
        "duolm_vid_table_load": (I, [VP, VP, I64]),
        "duolm_vid_table_build": (I, [VP, VP, I64, ctypes.c_double, ctypes.c_double]),
        "duolm_embedding_rho": (I, [VP, P(ctypes.c_double)]),
        "duolm_reserve": (I, [VP, I64, I64, I64]),
        "duolm_prepare": (I, [VP, I, VP, VP, VP, VP, I, I]),
        "duolm_execute": (I, [VP]),
        "duolm_scores_device": (VP, [VP]),
        "duolm_sync": (I, [VP]),
        "duolm_score": (I, [VP, I, VP, VP, VP, VP, I, I, VP]),
        "duolm_set_graph": (I, [VP, I]),
        "duolm_set_pdl": (I, [VP, I]),
        "duolm_launches_per_execute": (I64, [VP]),
        "duolm_last_error": (ctypes.c_char_p, [VP]),
        "duolm_destroy": (None, [VP]),
        "duolm_debug_layout": (I, [VP, P(I64), VP, VP]),
        "duolm_debug_mask": (I, [VP, I, VP]),
        "duolm_debug_residual": (I, [VP, I, VP]),
        "duolm_debug_table": (I, [VP, VP, I64]),
        "duolm_plan_bytes": (I64, [VP]),
        "duolm_debug_gemm": (I, [VP, I, I, VP, VP]),
        "duolm_profile": (I, [VP, I, VP, VP]),
        "duolm_debug_wait_timeout": (I, [VP]),
        "duolm_embedding_rho_static": (I, [VP, I, I64, I, VP, VP]),
        "duolm_gather": (I, [VP, VP, I64, VP, VP, VP]),
        "duolm_compile": (I, [P(Template), I, VP, VP, VP, VP, VP, VP, I64, I, VP, I64, VP, VP, I64]),
        "duolm_compile_append": (I, [P(Template), I, VP, VP, VP, VP, VP, VP, I64, I, VP, VP, I64, VP, VP, I64, VP,
                                     VP]),
        "duolm_debug_attention_plan": (I64, [I, VP, VP, VP, I, I, I, I, VP, I64, VP]),
        "duolm_kv_store_reserve": (I, [VP, I, I]),
        "duolm_kv_slot_length": (I, [VP, I]),
        "duolm_prepare_cached": (I, [VP, I, VP, VP, VP, VP, I, VP, VP, VP]),
        "duolm_score_cached": (I, [VP, I, VP, VP, VP, VP, I, VP, VP, VP, VP]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


RHO_STATIC_MAX_ROWS = 262144


def embedding_rho_static(embed_dev: int, dtype: int, vocab: int, d: int, rho_out_dev: int,
                         stream: Optional[int] = None) -> None:
    """duolm_embedding_rho_static: device pointers in, nothing allocated."""
    rc = lib.duolm_embedding_rho_static(ctypes.c_void_p(embed_dev), int(dtype), int(vocab), int(d),
                                        ctypes.c_void_p(rho_out_dev), ctypes.c_void_p(stream or 0))
    if rc != 0:
        raise DuolmError(rc, f"duolm_embedding_rho_static(vocab={vocab}, d={d}, dtype={dtype}) failed")


def compile_requests(vocab: int, marker: int, m: int, instr, header, branch_header, hist_items, hist_offsets,
                     feedback, feedback_offsets, cand_items, cand_offsets, n_items: int, n_threads: int = 0,
                     hist_cached=None):
    """duolm_compile: request records -> (prefix_ids, prefix_offsets,
    branch_ids, cand_offsets, branch_len), host arrays in the layout
    duolm_prepare / duolm_score take.  With hist_cached (per request: -1, or
    the history items its KV slot already holds), duolm_compile_append:
    the result also carries the cached and keep arrays of
    duolm_prepare_cached."""
    ins, hdr, bh = (np.ascontiguousarray(x, np.int32) for x in (instr, header, branch_header))
    tpl = Template(int(vocab), int(marker), int(m), ins.ctypes.data, len(ins), hdr.ctypes.data, len(hdr),
                   bh.ctypes.data, len(bh))
    hi, ho = np.ascontiguousarray(hist_items, np.int64), np.ascontiguousarray(hist_offsets, np.int64)
    fb, fo = np.ascontiguousarray(feedback, np.int32), np.ascontiguousarray(feedback_offsets, np.int64)
    ci, co = np.ascontiguousarray(cand_items, np.int64), np.ascontiguousarray(cand_offsets, np.int64)
    R = len(ho) - 1
    n_hist = np.diff(ho)
    cap = int(R * (len(ins) + len(hdr)) + n_hist.sum() * (1 + m) + len(fb))
    b = len(bh) + m
    prefix = np.empty(max(cap, 1), np.int32)
    poff = np.empty(R + 1, np.int64)
    branch = np.empty(max(int(co[-1]) * b, 1), np.int32)
    if hist_cached is None:
        rc = lib.duolm_compile(ctypes.byref(tpl), R, _p(hi), _p(ho), _p(fb), _p(fo), _p(ci), _p(co), int(n_items),
                               int(n_threads), _p(prefix), prefix.size, _p(poff), _p(branch), branch.size)
    else:
        hc = np.ascontiguousarray(hist_cached, np.int32)
        cached = np.zeros(R, np.int32)
        keep = np.zeros(R, np.int32)
        rc = lib.duolm_compile_append(ctypes.byref(tpl), R, _p(hi), _p(ho), _p(fb), _p(fo), _p(ci), _p(co),
                                      int(n_items), int(n_threads), _p(hc), _p(prefix), prefix.size, _p(poff),
                                      _p(branch), branch.size, _p(cached), _p(keep))
    if rc != 0:
        raise DuolmError(rc, lib.duolm_last_error(None).decode())
    out = (prefix[:int(poff[-1])], poff, branch[:int(co[-1]) * b], co, b)
    return out if hist_cached is None else out + (cached, keep)


def attention_plan(L, K, cached, branch_len: int, n_kv_heads: int, rows_per_item: int, n_ctas: int):
    """duolm_debug_attention_plan: (items [n][4], cta_off [n_ctas + 1])."""
    Ls, Ks, cs = (np.ascontiguousarray(x, np.int32) for x in (L, K, cached))
    per = (rows_per_item // branch_len) * branch_len
    cap = int(n_kv_heads * sum((k * branch_len + per - 1) // per + (l - c + rows_per_item - 1) // rows_per_item
                               for l, k, c in zip(Ls, Ks, cs)))
    items = np.zeros((max(cap, 1), 4), np.int32)
    cta = np.zeros(n_ctas + 1, np.int32)
    n = lib.duolm_debug_attention_plan(len(Ls), _p(Ls), _p(Ks), _p(cs), int(branch_len), int(n_kv_heads),
                                       int(rows_per_item), int(n_ctas), _p(items), cap, _p(cta))
    if n < 0:
        raise DuolmError(int(n), "duolm_debug_attention_plan")
    return items[:n], cta


def _arr(a, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a.size else ctypes.c_void_p(a.ctypes.data or 16)


class Ranker:
    """One library context (device memory, stream, CUDA graph) for one model."""

    def __init__(self, shape, weights: Sequence[np.ndarray], device: int = 0, stream: Optional[int] = None):
        """``shape`` has the fields of the C model descriptor (``n_layers, d,
        n_q_heads, n_kv_heads, head_dim, ffn, vocab, rope_theta, rms_eps``) and
        ``dtype`` ("bf16" or "fp32"); ``weights`` are the host tensors in load
        order (uint16 bfloat16 bits or float32); ``stream`` is a cudaStream_t
        handle (e.g. ``torch.cuda.current_stream().cuda_stream``) or None."""
        dt = DTYPE_BF16 if shape.dtype == "bf16" else DTYPE_FP32
        self.desc = ModelDesc(shape.n_layers, shape.d, shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                              shape.ffn, shape.vocab, shape.rope_theta, shape.rms_eps, dt)
        want = np.uint16 if dt == DTYPE_BF16 else np.float32
        n = lib.duolm_weight_count(ctypes.byref(self.desc))
        if n != len(weights):
            raise ValueError(f"expected {n} weight tensors, got {len(weights)}")
        self._keep = [_arr(w, want) for w in weights]
        ptrs = (ctypes.c_void_p * n)(*[w.ctypes.data for w in self._keep])
        ctx = ctypes.c_void_p()
        rc = lib.duolm_model_load(ctypes.byref(self.desc), ptrs, device, stream or None, ctypes.byref(ctx))
        self._keep = None
        if rc != 0:
            raise DuolmError(rc, lib.duolm_last_error(None).decode())
        self.ctx = ctx
        self.d = shape.d
        self.n_cand = 0

    def _check(self, rc: int):
        if rc != 0:
            raise DuolmError(rc, lib.duolm_last_error(self.ctx).decode())

    def close(self):
        if getattr(self, "ctx", None):
            lib.duolm_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- item table
    def vid_table_load(self, rows_fp16: np.ndarray):
        rows = _arr(np.asarray(rows_fp16).view(np.uint16) if np.asarray(rows_fp16).dtype == np.float16
                    else rows_fp16, np.uint16)
        self._check(lib.duolm_vid_table_load(self.ctx, _p(rows), rows.shape[0]))

    def vid_table_build(self, a_rows: np.ndarray, gamma: float, rho: float):
        a = _arr(a_rows, np.float32)
        self._check(lib.duolm_vid_table_build(self.ctx, _p(a), a.shape[0], float(gamma), float(rho)))

    def embedding_rho(self) -> float:
        v = ctypes.c_double()
        self._check(lib.duolm_embedding_rho(self.ctx, ctypes.byref(v)))
        return v.value

    # ---- batches
    def reserve(self, max_tokens: int, max_requests: int, max_candidates: int):
        self._check(lib.duolm_reserve(self.ctx, max_tokens, max_requests, max_candidates))

    def prepare(self, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len: int, mode: int = MODE_MIS):
        a = [_arr(prefix_ids, np.int32), _arr(prefix_offsets, np.int64), _arr(branch_ids, np.int32),
             _arr(cand_offsets, np.int64)]
        self._check(lib.duolm_prepare(self.ctx, a[1].shape[0] - 1, _p(a[0]), _p(a[1]), _p(a[2]), _p(a[3]),
                                      int(branch_len), int(mode)))
        self.n_cand = int(a[3][-1])

    def execute(self):
        self._check(lib.duolm_execute(self.ctx))

    def scores_device(self) -> int:
        return lib.duolm_scores_device(self.ctx)

    def sync(self):
        self._check(lib.duolm_sync(self.ctx))

    def score(self, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len: int,
              mode: int = MODE_MIS, out: Optional[np.ndarray] = None) -> np.ndarray:
        a = [_arr(prefix_ids, np.int32), _arr(prefix_offsets, np.int64), _arr(branch_ids, np.int32),
             _arr(cand_offsets, np.int64)]
        n = int(a[3][-1])
        if out is None:
            out = np.empty(n, np.float32)
        self._check(lib.duolm_score(self.ctx, a[1].shape[0] - 1, _p(a[0]), _p(a[1]), _p(a[2]), _p(a[3]),
                                    int(branch_len), int(mode), _p(out)))
        return out

    def score_workload(self, wl, mode: int = MODE_MIS) -> np.ndarray:
        p, po, b, co = wl.packed()
        return self.score(p, po, b, co, wl.branch_len, mode)

    # ---- prefix KV reuse
    def kv_store_reserve(self, n_slots: int, slot_tokens: int):
        self._check(lib.duolm_kv_store_reserve(self.ctx, int(n_slots), int(slot_tokens)))

    def kv_slot_length(self, slot: int) -> int:
        n = lib.duolm_kv_slot_length(self.ctx, int(slot))
        if n < 0:
            raise DuolmError(n, f"kv_slot_length({slot})")
        return n

    def _cached_args(self, prefix_ids, prefix_offsets, branch_ids, cand_offsets, slot, cached, keep):
        a = [_arr(prefix_ids, np.int32), _arr(prefix_offsets, np.int64), _arr(branch_ids, np.int32),
             _arr(cand_offsets, np.int64)]
        R = a[1].shape[0] - 1
        s = [_arr(np.broadcast_to(v, (R,)), np.int32) for v in (slot, cached, keep)]
        return a, s, R

    def prepare_cached(self, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len: int, slot, cached,
                       keep):
        """duolm_prepare_cached: request q continues the first cached[q]
        tokens slot[q] holds and appends keep[q] of its new prefix tokens."""
        a, s, R = self._cached_args(prefix_ids, prefix_offsets, branch_ids, cand_offsets, slot, cached, keep)
        self._check(lib.duolm_prepare_cached(self.ctx, R, _p(a[0]), _p(a[1]), _p(a[2]), _p(a[3]), int(branch_len),
                                             _p(s[0]), _p(s[1]), _p(s[2])))
        self.n_cand = int(a[3][-1])

    def score_cached(self, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len: int, slot, cached,
                     keep, out: Optional[np.ndarray] = None) -> np.ndarray:
        a, s, R = self._cached_args(prefix_ids, prefix_offsets, branch_ids, cand_offsets, slot, cached, keep)
        if out is None:
            out = np.empty(int(a[3][-1]), np.float32)
        self._check(lib.duolm_score_cached(self.ctx, R, _p(a[0]), _p(a[1]), _p(a[2]), _p(a[3]), int(branch_len),
                                           _p(s[0]), _p(s[1]), _p(s[2]), _p(out)))
        return out

    def set_graph(self, enabled: bool):
        self._check(lib.duolm_set_graph(self.ctx, 1 if enabled else 0))

    def set_pdl(self, enabled: bool):
        """Programmatic dependent launch between the pass's kernels (default on)."""
        self._check(lib.duolm_set_pdl(self.ctx, 1 if enabled else 0))

    def launches_per_execute(self) -> int:
        return int(lib.duolm_launches_per_execute(self.ctx))

    # ---- introspection
    def debug_layout(self):
        n = ctypes.c_int64()
        self._check(lib.duolm_debug_layout(self.ctx, ctypes.byref(n), None, None))
        ids = np.empty(n.value, np.int32)
        pos = np.empty(n.value, np.int32)
        self._check(lib.duolm_debug_layout(self.ctx, ctypes.byref(n), _p(ids), _p(pos)))
        return ids, pos

    def debug_mask(self, request: int, tq: int) -> np.ndarray:
        out = np.empty((tq, tq), np.uint8)
        self._check(lib.duolm_debug_mask(self.ctx, int(request), _p(out)))
        return out.astype(bool)

    def gather(self, ids_dev: int, n: int, x_dev: int, xg_dev: int, ssp_dev: int) -> None:
        """duolm_gather: the VID gather alone on device buffers (queued on the
        context's stream; sync() waits and checks the error flag)."""
        self._check(lib.duolm_gather(self.ctx, ctypes.c_void_p(ids_dev), int(n), ctypes.c_void_p(x_dev),
                                     ctypes.c_void_p(xg_dev), ctypes.c_void_p(ssp_dev)))

    def debug_residual(self, n_layers: int, n_tokens: int) -> np.ndarray:
        out = np.empty((n_tokens, self.d), np.float32)
        self._check(lib.duolm_debug_residual(self.ctx, int(n_layers), _p(out)))
        return out

    def plan_bytes(self) -> int:
        return int(lib.duolm_plan_bytes(self.ctx))

    PROFILE_CLASSES = ("embed", "gemm_qkv", "attention", "gemm_o", "rmsnorm", "gemm_gate_up", "gemm_down", "head",
                       "kv_append")

    def profile(self, n_steps: int) -> dict:
        """Per kernel class: (summed device ms over n_steps, launches)."""
        ms = np.zeros(len(self.PROFILE_CLASSES), np.float64)
        cnt = np.zeros(len(self.PROFILE_CLASSES), np.int64)
        self._check(lib.duolm_profile(self.ctx, int(n_steps), _p(ms), _p(cnt)))
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(self.PROFILE_CLASSES)}

    def debug_gemm(self, layer: int, which: int, a_fp16: np.ndarray, n_out: int) -> np.ndarray:
        a = _arr(np.asarray(a_fp16).view(np.uint16) if np.asarray(a_fp16).dtype == np.float16 else a_fp16,
                 np.uint16)
        out = np.empty((a.shape[0], n_out), np.float32)
        self._check(lib.duolm_debug_gemm(self.ctx, int(layer), int(which), _p(a), _p(out)))
        return out

    def debug_wait_timeout(self):
        self._check(lib.duolm_debug_wait_timeout(self.ctx))

    def debug_table(self, n_items: int) -> np.ndarray:
        out = np.empty((n_items, self.d), np.uint16)
        self._check(lib.duolm_debug_table(self.ctx, _p(out), int(n_items)))
        return out
