"""ctypes binding of the C ABI in ``include/mk.h`` (argument marshalling only).

Every computation runs in ``_lib/libmk.so``; this module only turns torch
tensors into device pointers and Python values into the ABI's structs.  There
is no fallback: a missing library or device raises.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Dict, List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmk.so")

MK_OK = 0
MK_ERR_INVALID_ARG = -1
MK_ERR_UNSUPPORTED = -2
MK_ERR_CUDA = -3
MK_ERR_RANGE = -4
MK_ERR_TIMEOUT = -5
MK_ERR_STATE = -6
MK_MAX_LAYERS = 128
MK_MAX_BATCH = 16
MODE_MEGAKERNEL = 0
MODE_PER_OP = 1
MODE_PER_OP_GRAPH = 2

ERROR_NAMES = {MK_OK: "MK_OK", MK_ERR_INVALID_ARG: "MK_ERR_INVALID_ARG",
               MK_ERR_UNSUPPORTED: "MK_ERR_UNSUPPORTED", MK_ERR_CUDA: "MK_ERR_CUDA",
               MK_ERR_RANGE: "MK_ERR_RANGE", MK_ERR_TIMEOUT: "MK_ERR_TIMEOUT",
               MK_ERR_STATE: "MK_ERR_STATE"}

#: every symbol include/mk.h declares
EXPORTS = ["mk_plan_create", "mk_plan_create_ex", "mk_decode_step", "mk_decode_step_ex",
           "mk_decode_step_host", "mk_plan_status", "mk_plan_error_info", "mk_plan_reset",
           "mk_plan_info", "mk_last_error", "mk_plan_destroy", "mk_decode_step_noalloc",
           "mk_plan_describe", "mk_plan_describe_schedule", "mk_prefill_chunk",
           "mk_w4_packed_bytes", "mk_w4_pack"]

#: bytes of the library's static scratch array used by mk_decode_step_noalloc
NOALLOC_SCRATCH_BYTES = 16 << 20


class mk_model_config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("hidden", C.c_int), ("n_q_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("vocab", C.c_int), ("rms_eps", C.c_float), ("rope_theta", C.c_float),
                ("qk_norm", C.c_int), ("max_seq_len", C.c_int)]


class mk_layer_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm",
                                           "wo", "mlp_norm", "w_gate", "w_up", "w_down")]


class mk_w4_layer_weights(C.Structure):
    _fields_ = [("q", C.c_void_p * 7)]


class mk_weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("layers", C.POINTER(mk_layer_weights)),
                ("final_norm", C.c_void_p), ("lm_head", C.c_void_p),
                ("w4_layers", C.POINTER(mk_w4_layer_weights))]


class mk_kv_cache(C.Structure):
    _fields_ = [("k_pages", C.POINTER(C.c_void_p)), ("v_pages", C.POINTER(C.c_void_p)),
                ("block_table", C.c_void_p), ("num_pages", C.c_int),
                ("max_pages_per_seq", C.c_int)]


class mk_plan_options(C.Structure):
    _fields_ = [("max_batch", C.c_int), ("kv_page_size", C.c_int), ("num_ctas", C.c_int),
                ("wait_limit_ns", C.c_int64), ("rows_per_task", C.c_int * 5),
                ("debug_unsatisfiable_dep", C.c_int), ("max_page_cols", C.c_int),
                ("o_split", C.c_int), ("gemv_path", C.c_int), ("schedule", C.c_int),
                ("weight_bits", C.c_int), ("prefill", C.c_int), ("attn_path", C.c_int)]


class mk_step_args(C.Structure):
    _fields_ = [("d_ids", C.c_void_p), ("d_pos", C.c_void_p), ("kv", C.POINTER(mk_kv_cache)),
                ("batch", C.c_int), ("d_out_ids", C.c_void_p), ("d_out_logits", C.c_void_p),
                ("d_out_pos", C.c_void_p), ("d_hidden", C.c_void_p), ("mode", C.c_int),
                ("d_trace", C.c_void_p)]


class mk_prefill_args(C.Structure):
    _fields_ = [("d_ids", C.c_void_p), ("n_tokens", C.c_int), ("pos0", C.c_int), ("seq", C.c_int),
                ("kv", C.POINTER(mk_kv_cache)), ("d_out_ids", C.c_void_p),
                ("d_out_logits", C.c_void_p), ("d_hidden", C.c_void_p), ("with_lm_head", C.c_int)]


class mk_plan_info_t(C.Structure):
    _fields_ = [("num_ctas", C.c_int), ("threads_per_cta", C.c_int), ("smem_bytes", C.c_int),
                ("n_pages", C.c_int), ("page_bytes", C.c_int), ("n_tasks", C.c_int),
                ("n_events", C.c_int), ("attn_slots", C.c_int),
                ("tokens_per_smem_page", C.c_int), ("rows_per_task", C.c_int * 5),
                ("page_cols", C.c_int * 4), ("weight_bytes", C.c_int64),
                ("events_per_layer", C.c_int), ("attn_slots_per_group", C.c_int),
                ("qkv_tasks_per_group", C.c_int), ("ffn_parts", C.c_int),
                ("ffn_part_cols", C.c_int), ("o_parts", C.c_int), ("o_part_cols", C.c_int),
                ("gemv_path", C.c_int), ("schedule", C.c_int), ("prefill", C.c_int),
                ("weight_bits", C.c_int), ("qkv_parts", C.c_int),
                ("gateup_parts", C.c_int), ("attn_path", C.c_int)]


_lib = None


def load_library(path: str = LIB_PATH) -> C.CDLL:
    """Load libmk.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"native library missing: {path} "
                           "(build it with `python -m persistent_task_runtime_b200.build`)")
    lib = C.CDLL(path)
    P = C.c_void_p
    lib.mk_plan_create.argtypes = [C.POINTER(mk_model_config), C.POINTER(mk_weights), C.c_int,
                                   C.c_int, C.POINTER(P)]
    lib.mk_plan_create_ex.argtypes = [C.POINTER(mk_model_config), C.POINTER(mk_weights),
                                      C.POINTER(mk_plan_options), C.POINTER(P)]
    lib.mk_decode_step.argtypes = [P, P, P, C.POINTER(mk_kv_cache), C.c_int, P, P, P]
    lib.mk_decode_step_ex.argtypes = [P, C.POINTER(mk_step_args), P]
    lib.mk_decode_step_host.argtypes = [P, P, P, C.POINTER(mk_kv_cache), C.c_int, P, P, P]
    lib.mk_plan_status.argtypes = [P]
    lib.mk_plan_error_info.argtypes = [P, C.POINTER(C.c_int32)]
    lib.mk_plan_reset.argtypes = [P]
    lib.mk_plan_info.argtypes = [P, C.POINTER(mk_plan_info_t)]
    lib.mk_plan_describe.argtypes = [C.POINTER(mk_model_config), C.POINTER(mk_plan_options),
                                     C.c_int, C.c_int, C.POINTER(mk_plan_info_t), P, C.c_int64]
    lib.mk_plan_describe_schedule.argtypes = [C.POINTER(mk_model_config),
                                              C.POINTER(mk_plan_options), C.c_int, C.c_int, P,
                                              C.c_int64]
    lib.mk_plan_describe_schedule.restype = C.c_int
    lib.mk_prefill_chunk.argtypes = [P, C.POINTER(mk_prefill_args), P]
    lib.mk_prefill_chunk.restype = C.c_int
    lib.mk_w4_packed_bytes.argtypes = [C.c_int, C.c_int]
    lib.mk_w4_packed_bytes.restype = C.c_int64
    lib.mk_w4_pack.argtypes = [P, P, C.c_int, C.c_int, P]
    lib.mk_w4_pack.restype = C.c_int
    lib.mk_last_error.restype = C.c_char_p
    lib.mk_last_error.argtypes = []
    lib.mk_plan_destroy.argtypes = [P]
    lib.mk_plan_destroy.restype = None
    lib.mk_decode_step_noalloc.argtypes = [C.POINTER(mk_model_config), C.POINTER(mk_weights),
                                           C.c_int, C.POINTER(mk_step_args), P]
    lib.mk_decode_step_noalloc.restype = C.c_int
    for name in ("mk_plan_create", "mk_plan_create_ex", "mk_decode_step", "mk_decode_step_ex",
                 "mk_decode_step_host", "mk_plan_status", "mk_plan_error_info",
                 "mk_plan_reset", "mk_plan_info"):
        getattr(lib, name).restype = C.c_int
    _lib = lib
    return lib


class MkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


def _check(rc: int):
    if rc != MK_OK:
        raise MkError(rc, load_library().mk_last_error().decode())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


class KVCacheView:
    """Host-side mk_kv_cache for a list of per-layer page tensors."""

    def __init__(self, k_pages: List[torch.Tensor], v_pages: List[torch.Tensor],
                 block_table: torch.Tensor):
        L = len(k_pages)
        self._tensors = (k_pages, v_pages, block_table)
        self._k = (C.c_void_p * L)(*[t.data_ptr() for t in k_pages])
        self._v = (C.c_void_p * L)(*[t.data_ptr() for t in v_pages])
        self.struct = mk_kv_cache(C.cast(self._k, C.POINTER(C.c_void_p)),
                                  C.cast(self._v, C.POINTER(C.c_void_p)),
                                  block_table.data_ptr(), k_pages[0].shape[0],
                                  block_table.shape[1])


#: one task record of mk_plan_describe (see include/mk.h)
TASK_RECORD_DTYPE = [("type", "u1"), ("n_m", "u1"), ("layer", "<u2"), ("row0", "<u4"),
                     ("nrows", "<u2"), ("ksplit", "u1"), ("nsplit", "u1"), ("dep_event", "<u4"),
                     ("dep_count", "<u4"), ("out_event", "<u4"), ("aux", "<u4"), ("aux2", "<u4"),
                     ("operands", "<u8", (3,)), ("map0", "<u4"), ("map1", "<u4")]
TASK_TYPES = {1: "embed", 2: "qkv", 3: "attn", 4: "oproj", 5: "gateup", 6: "down", 7: "lmhead"}
NO_EVENT = 0xFFFFFFFF


def _info_dict(i: "mk_plan_info_t") -> dict:
    out = {k: getattr(i, k) for k, _ in mk_plan_info_t._fields_}
    out["rows_per_task"] = list(i.rows_per_task)
    out["page_cols"] = list(i.page_cols)
    return out


def _config(cfg: Dict, max_seq_len: int) -> mk_model_config:
    return mk_model_config(cfg["n_layers"], cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"],
                           cfg["head_dim"], cfg["ffn"], cfg["vocab"], cfg.get("rms_eps", 1e-6),
                           cfg.get("rope_theta", 1e6), 1 if cfg.get("qk_norm", True) else 0,
                           max_seq_len)


def describe(cfg: Dict, max_batch: int = 1, page_size: int = 16, max_seq_len: int = 4096,
             num_sms: int = 148, smem_optin: int = 232448, rows_per_task=(0, 0, 0, 0, 0),
             max_page_cols: int = 0, o_split: bool = False, gemv_path: int = 0,
             schedule: int = 0, prefill: bool = False, weight_bits: int = 0,
             attn_path: int = 0):
    """The plan mk_plan_create_ex would build, without a GPU: (info, task records).

    The task records are a numpy structured array (TASK_RECORD_DTYPE)."""
    import numpy as np
    lib = load_library()
    c = _config(cfg, max_seq_len)
    opts = mk_plan_options(max_batch, page_size, 0, 0, (C.c_int * 5)(*rows_per_task), 0,
                           max_page_cols, 1 if o_split else 0, gemv_path, schedule, weight_bits,
                           1 if prefill else 0, attn_path)
    info = mk_plan_info_t()
    _check(lib.mk_plan_describe(C.byref(c), C.byref(opts), num_sms, smem_optin, C.byref(info),
                                None, 0))
    tasks = np.zeros(info.n_tasks, dtype=TASK_RECORD_DTYPE)
    assert tasks.itemsize == 64
    _check(lib.mk_plan_describe(C.byref(c), C.byref(opts), num_sms, smem_optin, C.byref(info),
                                tasks.ctypes.data, info.n_tasks))
    return _info_dict(info), tasks


def describe_schedule(cfg: Dict, n_tasks: int, max_batch: int = 1, page_size: int = 16,
                      max_seq_len: int = 4096, num_sms: int = 148, smem_optin: int = 232448,
                      gemv_path: int = 0, schedule: int = 1, rows_per_task=(0, 0, 0, 0, 0),
                      max_page_cols: int = 0, o_split: bool = False, prefill: bool = False,
                      weight_bits: int = 0, attn_path: int = 0):
    """CTA of every task under the plan's solidified schedule (-1: dynamic
    queue); the options are those of describe()."""
    import numpy as np
    lib = load_library()
    c = _config(cfg, max_seq_len)
    opts = mk_plan_options(max_batch, page_size, 0, 0, (C.c_int * 5)(*rows_per_task), 0,
                           max_page_cols, 1 if o_split else 0, gemv_path, schedule, weight_bits,
                           1 if prefill else 0, attn_path)
    out = np.zeros(n_tasks, dtype=np.int32)
    _check(lib.mk_plan_describe_schedule(C.byref(c), C.byref(opts), num_sms, smem_optin,
                                         out.ctypes.data, n_tasks))
    return out


W4_MATRIX_NAMES = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


def w4_pack(codes: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """mk_w4_pack on the host: codes uint8 [rows, cols] (0..15), scales bf16
    [rows, cols/128] -> the packed uint8 buffer the kernel streams (CPU)."""
    lib = load_library()
    rows, cols = codes.shape
    n = lib.mk_w4_packed_bytes(rows, cols)
    if n < 0:
        raise MkError(MK_ERR_INVALID_ARG, f"unsupported 4-bit matrix {rows} x {cols}")
    c = codes.detach().to("cpu", torch.uint8).contiguous()
    sc = scales.detach().to("cpu", torch.bfloat16).contiguous()
    out = torch.empty(n, dtype=torch.uint8)
    _check(lib.mk_w4_pack(c.data_ptr(), sc.data_ptr(), rows, cols, out.data_ptr()))
    return out


def _weight_structs(weights: Dict, L: int, device=None):
    """(mk_weights, keep-alive list): bf16 layers, plus packed 4-bit matrices
    on `device` when the layers carry ``w4`` (synth.make_w4_weights)."""
    keep = []
    lw = (mk_layer_weights * L)()
    w4 = "w4" in weights["layers"][0]
    for l, w in enumerate(weights["layers"]):
        lw[l] = mk_layer_weights(*[_ptr(w.get(k)) for k in (
            "attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm",
            "w_gate", "w_up", "w_down")])
    keep.append(lw)
    w4l = None
    if w4:
        dev = device or weights["embed"].device
        w4l = (mk_w4_layer_weights * L)()
        for l, w in enumerate(weights["layers"]):
            ptrs = []
            for name in W4_MATRIX_NAMES:
                codes, scales = w["w4"][name]
                packed = w4_pack(codes, scales).to(dev)
                keep.append(packed)
                ptrs.append(packed.data_ptr())
            w4l[l] = mk_w4_layer_weights((C.c_void_p * 7)(*ptrs))
        keep.append(w4l)
    mw = mk_weights(_ptr(weights["embed"]), lw, _ptr(weights["final_norm"]),
                    _ptr(weights["lm_head"]), w4l)
    return mw, keep


class Plan:
    """A decode plan over caller-owned bf16 weights (see include/mk.h)."""

    def __init__(self, cfg: Dict, weights: Dict, max_batch: int = 1, page_size: int = 16,
                 max_seq_len: int = 4096, num_ctas: int = 0, wait_limit_ns: int = 0,
                 rows_per_task: Sequence[int] = (0, 0, 0, 0, 0), debug_unsatisfiable_dep=False,
                 max_page_cols: int = 0, o_split: bool = False, gemv_path: int = 0,
                 schedule: int = 0, prefill: bool = False, attn_path: int = 0):
        lib = load_library()
        self.cfg = dict(cfg)
        self.max_batch = max_batch
        self._c = _config(cfg, max_seq_len)
        L = cfg["n_layers"]
        self._weights = weights  # keep the tensors alive
        self._w, self._keep = _weight_structs(weights, L)
        opts = mk_plan_options(max_batch, page_size, num_ctas, wait_limit_ns,
                               (C.c_int * 5)(*rows_per_task), 1 if debug_unsatisfiable_dep else 0,
                               max_page_cols, 1 if o_split else 0, gemv_path, schedule, 0,
                               1 if prefill else 0, attn_path)
        h = C.c_void_p()
        _check(lib.mk_plan_create_ex(C.byref(self._c), C.byref(self._w), C.byref(opts),
                                     C.byref(h)))
        self._h = h
        self._lib = lib

    def info(self) -> dict:
        i = mk_plan_info_t()
        _check(self._lib.mk_plan_info(self._h, C.byref(i)))
        return _info_dict(i)

    def step(self, ids: torch.Tensor, pos: torch.Tensor, kv: KVCacheView, out_ids: torch.Tensor,
             out_logits: Optional[torch.Tensor] = None, out_pos: Optional[torch.Tensor] = None,
             hidden: Optional[torch.Tensor] = None, mode: int = MODE_MEGAKERNEL,
             batch: Optional[int] = None, trace: Optional[torch.Tensor] = None,
             stream=None) -> None:
        """Enqueue one decode step (asynchronous; see status())."""
        b = ids.shape[0] if batch is None else batch
        a = mk_step_args(_ptr(ids), _ptr(pos), C.pointer(kv.struct), b, _ptr(out_ids),
                         _ptr(out_logits), _ptr(out_pos), _ptr(hidden), mode, _ptr(trace))
        _check(self._lib.mk_decode_step_ex(self._h, C.byref(a), _stream_handle(stream)))

    def prefill_chunk(self, ids: torch.Tensor, pos0: int, seq: int, kv: KVCacheView,
                      out_ids: Optional[torch.Tensor] = None,
                      out_logits: Optional[torch.Tensor] = None,
                      hidden: Optional[torch.Tensor] = None, with_lm_head: bool = True,
                      stream=None) -> None:
        """mk_prefill_chunk: tokens ids[0..n) of sequence `seq` at positions
        pos0.. as one launch (asynchronous; see status())."""
        a = mk_prefill_args(_ptr(ids), ids.shape[0], pos0, seq, C.pointer(kv.struct),
                            _ptr(out_ids), _ptr(out_logits), _ptr(hidden),
                            1 if with_lm_head else 0)
        _check(self._lib.mk_prefill_chunk(self._h, C.byref(a), _stream_handle(stream)))

    def prefill(self, prompt: torch.Tensor, seq: int, kv: KVCacheView, out_ids: torch.Tensor,
                chunk: Optional[int] = None, stream=None) -> None:
        """A whole prompt (device int32 ids) of sequence `seq` from position 0,
        in chunks of `chunk` tokens (default: max_batch); the LM head runs on
        the last chunk only.  out_ids[0] receives the first generated token."""
        n = prompt.shape[0]
        T = chunk or self.max_batch
        for p0 in range(0, n, T):
            m = min(T, n - p0)
            last = p0 + m == n
            self.prefill_chunk(prompt[p0:p0 + m], p0, seq, kv,
                               out_ids=self._chunk_out(m) if last else None,
                               with_lm_head=last, stream=stream)
            if last:
                out_ids.copy_(self._chunk_ids[m - 1:m])

    def _chunk_out(self, m):
        if getattr(self, "_chunk_ids", None) is None:
            self._chunk_ids = torch.zeros(self.max_batch, dtype=torch.int32, device="cuda")
        return self._chunk_ids[:m]

    def step_plain(self, ids, pos, kv: KVCacheView, batch, out_ids, out_logits=None,
                   stream=None) -> None:
        """The six-argument mk_decode_step entry point."""
        _check(self._lib.mk_decode_step(self._h, _ptr(ids), _ptr(pos), C.pointer(kv.struct),
                                        batch, _ptr(out_ids), _ptr(out_logits),
                                        _stream_handle(stream)))

    def step_host(self, h_ids: torch.Tensor, h_pos: torch.Tensor, kv: KVCacheView,
                  h_out_ids: torch.Tensor, h_out_logits: Optional[torch.Tensor] = None,
                  stream=None) -> int:
        """mk_decode_step_host: host buffers in and out; returns the device status."""
        rc = self._lib.mk_decode_step_host(self._h, _ptr(h_ids), _ptr(h_pos), C.pointer(kv.struct),
                                           h_ids.shape[0], _ptr(h_out_ids), _ptr(h_out_logits),
                                           _stream_handle(stream))
        if rc in (MK_ERR_INVALID_ARG, MK_ERR_UNSUPPORTED, MK_ERR_CUDA):
            _check(rc)
        return rc

    def status(self) -> int:
        return self._lib.mk_plan_status(self._h)

    def error_info(self) -> List[int]:
        buf = (C.c_int32 * 4)()
        _check(self._lib.mk_plan_error_info(self._h, buf))
        return list(buf)

    def reset(self) -> None:
        _check(self._lib.mk_plan_reset(self._h))

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.mk_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def decode_step_noalloc(plan_like: "Plan", ids: torch.Tensor, pos: torch.Tensor, kv: KVCacheView,
                        out_ids: torch.Tensor, out_logits: Optional[torch.Tensor] = None,
                        page_size: int = 16, stream=None,
                        trace: Optional[torch.Tensor] = None) -> int:
    """mk_decode_step_noalloc: one step with no device allocation by the library.

    ``plan_like`` only supplies the model config and weight pointers (its
    ctypes structs); the call does not use the plan's device memory.  Returns
    the device status (raises on host-side errors)."""
    lib = load_library()
    a = mk_step_args(_ptr(ids), _ptr(pos), C.pointer(kv.struct), ids.shape[0], _ptr(out_ids),
                     _ptr(out_logits), None, None, MODE_MEGAKERNEL, _ptr(trace))
    rc = lib.mk_decode_step_noalloc(C.byref(plan_like._c), C.byref(plan_like._w), page_size,
                                    C.byref(a), _stream_handle(stream))
    if rc in (MK_ERR_INVALID_ARG, MK_ERR_UNSUPPORTED, MK_ERR_CUDA):
        _check(rc)
    return rc


class ModelRef:
    """The config and weight-pointer structs of a model, without a plan (for
    mk_decode_step_noalloc)."""

    def __init__(self, cfg: Dict, weights: Dict, max_seq_len: int = 4096):
        self._c = _config(cfg, max_seq_len)
        L = cfg["n_layers"]
        self._weights = weights
        self._w, self._keep = _weight_structs(weights, L)
