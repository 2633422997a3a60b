"""Python binding of libdms (ctypes): argument marshalling only.

Every function mirrors one C entry point of ``include/dms.h`` /
``include/dms_synth.h`` under the same name and returns what the C call
writes.  A non-OK status raises ``DmsError`` carrying the status and the
library's last error message.  Tensors are passed as raw pointers; PyTorch
is used only for device memory and streams (``Pool`` allocates the pool
buffer with it).  Importing this module does not load the library; the first
call does, and it raises ``DmsLibraryMissing`` when ``libdms.so`` has not
been built -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# DMS_LIBRARY=debug selects libdms_debug.so (device bounds checks, DMS_DEBUG)
LIB_PATH = os.path.join(_HERE, "libdms_debug.so" if os.environ.get("DMS_LIBRARY") == "debug"
                        else "libdms.so")

DMS_OK, DMS_ERR_INVALID_ARG, DMS_ERR_CAPACITY, DMS_ERR_CUDA, DMS_ERR_UNSUPPORTED, DMS_ERR_DEVICE = range(6)
DMS_F32, DMS_BF16, DMS_FP8_E4M3, DMS_INT4 = 0, 1, 2, 3

DEVERR_BLOCKS_EXHAUSTED = 0x1
DEVERR_HEAD_TABLE_FULL = 0x2
DEVERR_FREE_STACK_FULL = 0x4
DEVERR_TIMEOUT = 0x8
DEVERR_LAYER_NOT_EMPTY = 0x10
DEVERR_BOUNDS = 0x20
DEVERR_BAD_SEQUENCE = 0x40

FAULT_DROP_INPUT_SIGNAL = 1
ATTN_AUTO, ATTN_STREAM_K, ATTN_CLUSTER = 0, 1, 2
PREFILL_SPARSE, PREFILL_DENSE = 0, 1

BLOCK_TOKENS = 64


class DmsLibraryMissing(RuntimeError):
    pass


class DmsError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {msg}")


class PoolConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("max_batch", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32),
                ("block_tokens", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("max_blocks", ctypes.c_int64), ("max_context", ctypes.c_int64)]


class PoolLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in
                ("header", "blocks", "block_table", "n_slots", "n_retained", "ring", "ring_row",
                 "last_block", "free_top", "free_stack", "block_stack", "scales", "tickets",
                 "scratch", "total")] + [
        ("block_bytes", ctypes.c_int64), ("row_bytes", ctypes.c_int64),
        ("max_blocks_per_head", ctypes.c_int32), ("free_stack_cap", ctypes.c_int32),
        ("n_heads", ctypes.c_int32), ("fp8_layout", ctypes.c_int32)]


class PoolStats(ctypes.Structure):
    _fields_ = [("retained_tokens", ctypes.c_int64), ("slots_in_use", ctypes.c_int64),
                ("min_retained", ctypes.c_int32), ("max_retained", ctypes.c_int32),
                ("heads_nonempty", ctypes.c_int32), ("pad0", ctypes.c_int32),
                ("blocks_in_use", ctypes.c_int64), ("blocks_total", ctypes.c_int64),
                ("kv_bytes_in_use", ctypes.c_int64), ("kv_bytes_retained", ctypes.c_int64),
                ("error_flags", ctypes.c_uint32), ("error_layer", ctypes.c_int32),
                ("error_seq", ctypes.c_int32), ("error_head", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_ if f != "pad0"}


class StepperLayout(ctypes.Structure):
    _fields_ = [("k", ctypes.c_size_t), ("v", ctypes.c_size_t), ("q", ctypes.c_size_t),
                ("evict", ctypes.c_size_t), ("in_bytes", ctypes.c_size_t),
                ("out_bytes", ctypes.c_size_t), ("device_bytes", ctypes.c_size_t)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SIGS = {
    "dms_status_string": (ctypes.c_char_p, [_I]),
    "dms_last_error": (ctypes.c_char_p, []),
    "dms_pool_bytes_required": (_I, [ctypes.POINTER(PoolConfig), ctypes.POINTER(ctypes.c_size_t)]),
    "dms_pool_create": (_I, [ctypes.POINTER(PoolConfig), _P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]),
    "dms_pool_destroy": (_I, [_P]),
    "dms_pool_reset": (_I, [_P, _P]),
    "dms_pool_layout": (_I, [_P, ctypes.POINTER(PoolLayout)]),
    "dms_pool_set_wait_limit": (_I, [_P, ctypes.c_uint64]),
    "dms_pool_set_attn_kernel": (_I, [_P, _I]),
    "dms_pool_set_prefill_mode": (_I, [_P, _I]),
    "dms_decode_attn_plan": (_I, [_P, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "dms_decode_step_layers": (_I, [_P, _I, _I, _I, _I64, _P, _P, _I, _P, _P, _I, _P, ctypes.c_float, _P,
                                    ctypes.c_size_t, _P]),
    "dms_stepper_inject_fault": (_I, [_P, _I]),
    "dms_compact_prefill": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P]),
    "dms_append_evict_layers": (_I, [_P, _I, _I, _I, _I64, _P, _P, _I, _P, _P]),
    "dms_append_evict": (_I, [_P, _I, _I, _I64, _P, _P, _I, _P, _P]),
    "dms_decode_workspace_bytes": (_I, [_P, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "dms_decode_attn_layers": (_I, [_P, _I, _I, _I, _P, _I, _P, ctypes.c_float, _P, ctypes.c_size_t, _P]),
    "dms_decode_attn": (_I, [_P, _I, _I, _P, _I, _P, ctypes.c_float, _P, ctypes.c_size_t, _P]),
    "dms_decode_attn_layers_noalloc": (_I, [_P, _I, _I, _I, _P, _I, _P, ctypes.c_float, _P]),
    "dms_pool_stats": (_I, [_P, ctypes.POINTER(PoolStats), _P]),
    "dms_compact_prefill_seqs": (_I, [_P, _I, _I, _I, _I, _P, _P, _I, _P, _P]),
    "dms_append_evict_seqs": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P]),
    "dms_decode_attn_seqs": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, ctypes.c_float, _P, ctypes.c_size_t, _P]),
    "dms_release_seqs": (_I, [_P, _I, _P, _P]),
    "dms_prefill_attn": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _P, ctypes.c_float, _P]),
    "dms_project_workspace_bytes": (_I, [_P, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "dms_project_append": (_I, [_P, _I, _I, _P, _P, _P, _I, _P, _P, _P, ctypes.c_float, _P, ctypes.c_size_t, _P]),
    "dms_stepper_layout": (_I, [_P, _I, _I, ctypes.POINTER(StepperLayout)]),
    "dms_stepper_create": (_I, [_P, _I, _I, _I, ctypes.c_float, _P, ctypes.c_size_t, _P, ctypes.POINTER(_P)]),
    "dms_stepper_step": (_I, [_P, _I64, _P, _P]),
    "dms_stepper_join": (_I, [_P, _P]),
    "dms_stepper_destroy": (_I, [_P]),
    "dms_synth_normal": (_I, [ctypes.c_uint64, _I, _I, _I, _I, _I64, _I, _I, _I, _I, _P, _P]),
    "dms_synth_flags": (_I, [ctypes.c_uint64, _I, _I, _I, _I64, _I, _I, _P, _P, _P]),
}
EXPORTED = sorted(_SIGS)

_lib = None


def lib() -> ctypes.CDLL:
    """Load libdms.so (once).  Raises DmsLibraryMissing if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DmsLibraryMissing(
                f"{LIB_PATH} not built; run `python -m compact_decode_attention_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def _check(status: int, where: str):
    if status != DMS_OK:
        msg = lib().dms_last_error().decode(errors="replace")
        raise DmsError(status, where, msg)


def dms_status_string(s: int) -> str:
    return lib().dms_status_string(s).decode()


def dms_pool_bytes_required(cfg: PoolConfig) -> int:
    n = ctypes.c_size_t()
    _check(lib().dms_pool_bytes_required(ctypes.byref(cfg), ctypes.byref(n)), "dms_pool_bytes_required")
    return n.value


def dms_pool_create(cfg: PoolConfig, dev_buf: int, nbytes: int, stream: int) -> int:
    h = _P()
    _check(lib().dms_pool_create(ctypes.byref(cfg), dev_buf, nbytes, stream, ctypes.byref(h)),
           "dms_pool_create")
    return h.value


def dms_pool_destroy(pool: int):
    _check(lib().dms_pool_destroy(pool), "dms_pool_destroy")


def dms_pool_reset(pool: int, stream: int):
    _check(lib().dms_pool_reset(pool, stream), "dms_pool_reset")


def dms_pool_set_wait_limit(pool: int, limit_ns: int):
    _check(lib().dms_pool_set_wait_limit(pool, limit_ns), "dms_pool_set_wait_limit")


def dms_pool_set_attn_kernel(pool: int, kind: int):
    _check(lib().dms_pool_set_attn_kernel(pool, kind), "dms_pool_set_attn_kernel")


def dms_pool_set_prefill_mode(pool: int, mode: int):
    _check(lib().dms_pool_set_prefill_mode(pool, mode), "dms_pool_set_prefill_mode")


def dms_decode_attn_plan(pool: int, n_layers: int, batch: int) -> tuple:
    """(kernel, cluster_size) a decode attention call over n_layers x batch would use."""
    k, c = _I(), _I()
    _check(lib().dms_decode_attn_plan(pool, n_layers, batch, ctypes.byref(k), ctypes.byref(c)),
           "dms_decode_attn_plan")
    return k.value, c.value


def dms_decode_step_layers(pool: int, layer0: int, n_layers: int, batch: int, pos: int, k: int, v: int,
                           in_dtype: int, evict: int, q: int, q_dtype: int, out: int, sm_scale: float,
                           workspace: int, workspace_bytes: int, stream: int):
    _check(lib().dms_decode_step_layers(pool, layer0, n_layers, batch, pos, k, v, in_dtype, evict, q,
                                        q_dtype, out, sm_scale, workspace, workspace_bytes, stream),
           "dms_decode_step_layers")


def dms_stepper_inject_fault(st: int, fault: int):
    _check(lib().dms_stepper_inject_fault(st, fault), "dms_stepper_inject_fault")


def dms_pool_layout(pool: int) -> PoolLayout:
    lay = PoolLayout()
    _check(lib().dms_pool_layout(pool, ctypes.byref(lay)), "dms_pool_layout")
    return lay


def dms_compact_prefill(pool: int, layer: int, batch: int, prompt_len: int, k: int, v: int,
                        in_dtype: int, evict: int, stream: int):
    _check(lib().dms_compact_prefill(pool, layer, batch, prompt_len, k, v, in_dtype, evict, stream),
           "dms_compact_prefill")


def dms_append_evict_layers(pool: int, layer0: int, n_layers: int, batch: int, pos: int, k: int,
                            v: int, in_dtype: int, evict: int, stream: int):
    _check(lib().dms_append_evict_layers(pool, layer0, n_layers, batch, pos, k, v, in_dtype, evict,
                                         stream), "dms_append_evict_layers")


def dms_append_evict(pool: int, layer: int, batch: int, pos: int, k: int, v: int, in_dtype: int,
                     evict: int, stream: int):
    _check(lib().dms_append_evict(pool, layer, batch, pos, k, v, in_dtype, evict, stream),
           "dms_append_evict")


def dms_decode_workspace_bytes(pool: int, n_layers: int, batch: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().dms_decode_workspace_bytes(pool, n_layers, batch, ctypes.byref(n)),
           "dms_decode_workspace_bytes")
    return n.value


def dms_decode_attn_layers(pool: int, layer0: int, n_layers: int, batch: int, q: int, q_dtype: int,
                           out: int, sm_scale: float, workspace: int, workspace_bytes: int,
                           stream: int):
    _check(lib().dms_decode_attn_layers(pool, layer0, n_layers, batch, q, q_dtype, out, sm_scale,
                                        workspace, workspace_bytes, stream), "dms_decode_attn_layers")


def dms_decode_attn(pool: int, layer: int, batch: int, q: int, q_dtype: int, out: int,
                    sm_scale: float, workspace: int, workspace_bytes: int, stream: int):
    _check(lib().dms_decode_attn(pool, layer, batch, q, q_dtype, out, sm_scale, workspace,
                                 workspace_bytes, stream), "dms_decode_attn")


def dms_decode_attn_layers_noalloc(pool: int, layer0: int, n_layers: int, batch: int, q: int,
                                   q_dtype: int, out: int, sm_scale: float, stream: int):
    _check(lib().dms_decode_attn_layers_noalloc(pool, layer0, n_layers, batch, q, q_dtype, out,
                                                sm_scale, stream), "dms_decode_attn_layers_noalloc")


def dms_pool_stats(pool: int, stream: int, check: bool = True) -> PoolStats:
    st = PoolStats()
    rc = lib().dms_pool_stats(pool, ctypes.byref(st), stream)
    if check:
        _check(rc, "dms_pool_stats")
    return st


def dms_compact_prefill_seqs(pool: int, layer: int, seq0: int, batch: int, prompt_len: int, k: int,
                             v: int, in_dtype: int, evict: int, stream: int):
    _check(lib().dms_compact_prefill_seqs(pool, layer, seq0, batch, prompt_len, k, v, in_dtype, evict,
                                          stream), "dms_compact_prefill_seqs")


def dms_append_evict_seqs(pool: int, layer0: int, n_layers: int, n_seqs: int, seq_ids: int, pos: int,
                          k: int, v: int, in_dtype: int, evict: int, stream: int):
    _check(lib().dms_append_evict_seqs(pool, layer0, n_layers, n_seqs, seq_ids, pos, k, v, in_dtype,
                                       evict, stream), "dms_append_evict_seqs")


def dms_decode_attn_seqs(pool: int, layer0: int, n_layers: int, n_seqs: int, seq_ids: int, q: int,
                         q_dtype: int, out: int, sm_scale: float, workspace: int, workspace_bytes: int,
                         stream: int):
    _check(lib().dms_decode_attn_seqs(pool, layer0, n_layers, n_seqs, seq_ids, q, q_dtype, out, sm_scale,
                                      workspace, workspace_bytes, stream), "dms_decode_attn_seqs")


def dms_prefill_attn(pool: int, layer: int, seq0: int, batch: int, prompt_len: int, q: int, k: int, v: int,
                     in_dtype: int, evict: int, out: int, sm_scale: float, stream: int):
    _check(lib().dms_prefill_attn(pool, layer, seq0, batch, prompt_len, q, k, v, in_dtype, evict, out,
                                  sm_scale, stream), "dms_prefill_attn")


def dms_project_workspace_bytes(pool: int, n_seqs: int, d_model: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().dms_project_workspace_bytes(pool, n_seqs, d_model, ctypes.byref(n)),
           "dms_project_workspace_bytes")
    return n.value


def dms_project_append(pool: int, layer: int, n_seqs: int, seq_ids: int, pos: int, x: int, d_model: int,
                       w_kv: int, w_evict: int, b_evict: int, threshold: float, workspace: int,
                       workspace_bytes: int, stream: int):
    _check(lib().dms_project_append(pool, layer, n_seqs, seq_ids, pos, x, d_model, w_kv, w_evict, b_evict,
                                    threshold, workspace, workspace_bytes, stream), "dms_project_append")


def dms_release_seqs(pool: int, n_seqs: int, seq_ids: int, stream: int):
    _check(lib().dms_release_seqs(pool, n_seqs, seq_ids, stream), "dms_release_seqs")


def dms_stepper_layout(pool: int, n_layers: int, batch: int) -> StepperLayout:
    lay = StepperLayout()
    _check(lib().dms_stepper_layout(pool, n_layers, batch, ctypes.byref(lay)), "dms_stepper_layout")
    return lay


def dms_stepper_create(pool: int, layer0: int, n_layers: int, batch: int, sm_scale: float,
                       device_buf: int, device_bytes: int, stream: int) -> int:
    h = _P()
    _check(lib().dms_stepper_create(pool, layer0, n_layers, batch, sm_scale, device_buf, device_bytes,
                                    stream, ctypes.byref(h)), "dms_stepper_create")
    return h.value


def dms_stepper_step(st: int, pos: int, host_in: int, host_out: int):
    _check(lib().dms_stepper_step(st, pos, host_in, host_out), "dms_stepper_step")


def dms_stepper_join(st: int, stream: int):
    _check(lib().dms_stepper_join(st, stream), "dms_stepper_join")


def dms_stepper_destroy(st: int):
    _check(lib().dms_stepper_destroy(st), "dms_stepper_destroy")


def dms_synth_normal(seed: int, stream_id: int, layer0: int, n_layers: int, batch: int, pos0: int,
                     n_pos: int, n_heads: int, head_dim: int, dtype: int, out: int, stream: int):
    _check(lib().dms_synth_normal(seed, stream_id, layer0, n_layers, batch, pos0, n_pos, n_heads,
                                  head_dim, dtype, out, stream), "dms_synth_normal")


def dms_synth_flags(seed: int, layer0: int, n_layers: int, batch: int, pos0: int, n_pos: int,
                    n_heads: int, thr: int, out: int, stream: int):
    _check(lib().dms_synth_flags(seed, layer0, n_layers, batch, pos0, n_pos, n_heads, thr, out,
                                 stream), "dms_synth_flags")


# ---------------------------------------------------------------------------
# torch plumbing: device memory and streams only
# ---------------------------------------------------------------------------

def torch_dtype_code(dtype) -> int:
    import torch
    if dtype == torch.float32:
        return DMS_F32
    if dtype == torch.bfloat16:
        return DMS_BF16
    raise ValueError(f"unsupported dtype {dtype}")


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return int(t.data_ptr())


class Pool:
    """A pool whose buffer is a torch uint8 CUDA tensor (owned by this object)."""

    def __init__(self, n_layers, max_batch, n_q_heads, n_kv_heads, head_dim, window, kv_dtype,
                 max_blocks, max_context, device="cuda", stream=None):
        import torch
        self.cfg = PoolConfig(n_layers, max_batch, n_q_heads, n_kv_heads, head_dim, window,
                              BLOCK_TOKENS, kv_dtype, max_blocks, max_context)
        self.nbytes = dms_pool_bytes_required(self.cfg)
        self.buffer = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        self.handle = dms_pool_create(self.cfg, _ptr(self.buffer), self.nbytes, _stream(stream))
        self.layout = dms_pool_layout(self.handle)
        self._ws = {}

    def close(self):
        if self.handle:
            dms_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reset(self, stream=None):
        dms_pool_reset(self.handle, _stream(stream))

    def set_wait_limit(self, limit_ns: int):
        dms_pool_set_wait_limit(self.handle, int(limit_ns))

    def set_attn_kernel(self, kind: int):
        dms_pool_set_attn_kernel(self.handle, int(kind))

    def set_prefill_mode(self, mode: int):
        dms_pool_set_prefill_mode(self.handle, int(mode))

    def compact_prefill(self, layer, k, v, evict, stream=None):
        B, P = k.shape[0], k.shape[1]
        dms_compact_prefill(self.handle, layer, B, P, _ptr(k), _ptr(v), torch_dtype_code(k.dtype),
                            _ptr(evict), _stream(stream))

    def append_evict_layers(self, layer0, pos, k, v, evict, stream=None):
        nl, B = k.shape[0], k.shape[1]
        dms_append_evict_layers(self.handle, layer0, nl, B, pos, _ptr(k), _ptr(v),
                                torch_dtype_code(k.dtype), _ptr(evict), _stream(stream))

    def workspace(self, n_layers, batch, device="cuda"):
        import torch
        key = (n_layers, batch)
        if key not in self._ws:
            n = dms_decode_workspace_bytes(self.handle, n_layers, batch)
            self._ws[key] = torch.empty(n, dtype=torch.uint8, device=device)
        return self._ws[key]

    def decode_attn_layers(self, layer0, q, out, sm_scale=0.0, stream=None):
        nl, B = q.shape[0], q.shape[1]
        ws = self.workspace(nl, B, q.device)
        dms_decode_attn_layers(self.handle, layer0, nl, B, _ptr(q), torch_dtype_code(q.dtype),
                               _ptr(out), sm_scale, _ptr(ws), ws.numel(), _stream(stream))

    def decode_step_layers(self, layer0, pos, k, v, evict, q, out, sm_scale=0.0, stream=None):
        """Append (k, v, evict [nl, B, Hkv(, D)]) then attend (q, out [nl, B, Hq, D]) in one call."""
        nl, B = q.shape[0], q.shape[1]
        ws = self.workspace(nl, B, q.device)
        dms_decode_step_layers(self.handle, layer0, nl, B, pos, _ptr(k), _ptr(v), torch_dtype_code(k.dtype),
                               _ptr(evict), _ptr(q), torch_dtype_code(q.dtype), _ptr(out), sm_scale, _ptr(ws),
                               ws.numel(), _stream(stream))

    # ---- continuous batching: sequence slots with their own positions ----
    def compact_prefill_seqs(self, layer, seq0, k, v, evict, stream=None):
        B, P = k.shape[0], k.shape[1]
        dms_compact_prefill_seqs(self.handle, layer, seq0, B, P, _ptr(k), _ptr(v),
                                 torch_dtype_code(k.dtype), _ptr(evict), _stream(stream))

    def append_evict_seqs(self, layer0, seq_ids, pos, k, v, evict, stream=None):
        """seq_ids int32 [n], pos int64 [n] (device); k, v [nl, n, Hkv, D]."""
        nl, n = k.shape[0], k.shape[1]
        dms_append_evict_seqs(self.handle, layer0, nl, n, _ptr(seq_ids), _ptr(pos), _ptr(k), _ptr(v),
                              torch_dtype_code(k.dtype), _ptr(evict), _stream(stream))

    def decode_attn_seqs(self, layer0, seq_ids, q, out, sm_scale=0.0, stream=None):
        nl, n = q.shape[0], q.shape[1]
        ws = self.workspace(nl, n, q.device)
        dms_decode_attn_seqs(self.handle, layer0, nl, n, _ptr(seq_ids), _ptr(q), torch_dtype_code(q.dtype),
                             _ptr(out), sm_scale, _ptr(ws), ws.numel(), _stream(stream))

    def prefill_attn(self, layer, seq0, q, k, v, evict, out, sm_scale=0.0, stream=None):
        """Prompt attention [B, P, Hq, D] under the DMS mask + compaction of the layer."""
        B, P = k.shape[0], k.shape[1]
        dms_prefill_attn(self.handle, layer, seq0, B, P, _ptr(q), _ptr(k), _ptr(v), torch_dtype_code(k.dtype),
                         _ptr(evict), _ptr(out), sm_scale, _stream(stream))

    def project_append(self, layer, seq_ids, pos, x, w_kv, w_evict, b_evict=None, threshold=0.0, stream=None):
        """x [n, d_model] bf16; appends one projected token per sequence (seq_ids may be None)."""
        import torch
        n, dm = x.shape
        key = ("proj", n, dm)
        if key not in self._ws:
            nb = dms_project_workspace_bytes(self.handle, n, dm)
            self._ws[key] = torch.empty(max(nb, 16), dtype=torch.uint8, device=x.device)
        ws = self._ws[key]
        dms_project_append(self.handle, layer, n, 0 if seq_ids is None else _ptr(seq_ids), _ptr(pos), _ptr(x), dm,
                           _ptr(w_kv), _ptr(w_evict), 0 if b_evict is None else _ptr(b_evict), threshold,
                           _ptr(ws), ws.numel(), _stream(stream))

    def release_seqs(self, seq_ids, stream=None):
        dms_release_seqs(self.handle, int(seq_ids.numel()), _ptr(seq_ids), _stream(stream))

    def stats(self, stream=None, check=True) -> PoolStats:
        return dms_pool_stats(self.handle, _stream(stream), check)

    # raw views of the bookkeeping regions (for tests and tools)
    def region(self, name, dtype, count):
        import torch
        off = getattr(self.layout, name)
        esz = torch.empty(0, dtype=dtype).element_size()
        return self.buffer[off: off + count * esz].view(dtype)


class Stepper:
    """Decode steps fed from pinned host memory (dms_stepper_*): one call per
    step enqueues the input copy, append/evict, decode attention and the
    output copy, pipelined against the neighbouring steps."""

    def __init__(self, pool: Pool, layer0, n_layers, batch, sm_scale=0.0, stream=None):
        import torch
        self.pool = pool
        self.layout = dms_stepper_layout(pool.handle, n_layers, batch)
        self.buffer = torch.empty(self.layout.device_bytes, dtype=torch.uint8, device=pool.buffer.device)
        self.stream = _stream(stream)
        self.handle = dms_stepper_create(pool.handle, layer0, n_layers, batch, sm_scale,
                                         _ptr(self.buffer), self.layout.device_bytes, self.stream)
        self._step = lib().dms_stepper_step
        self.n_layers, self.batch = n_layers, batch

    def host_inputs(self, n_steps: int):
        """Pinned uint8 host buffer for n_steps packed step inputs."""
        import torch
        return torch.empty(n_steps, self.layout.in_bytes, dtype=torch.uint8).pin_memory()

    def pack(self, dst, k, v, q, evict):
        """Write one step's inputs (torch tensors, any device) into the packed
        host row dst (uint8, layout.in_bytes)."""
        lay = self.layout
        for off, t in ((lay.k, k), (lay.v, v), (lay.q, q), (lay.evict, evict)):
            b = t.contiguous().view(-1).view(dtype=__import__("torch").uint8)
            dst[off: off + b.numel()].copy_(b)

    def step(self, pos, host_in, host_out):
        rc = self._step(self.handle, pos, host_in.data_ptr(), host_out.data_ptr())
        if rc != DMS_OK:
            _check(rc, "dms_stepper_step")

    def join(self, stream=None):
        dms_stepper_join(self.handle, _stream(stream))

    def inject_fault(self, fault: int):
        dms_stepper_inject_fault(self.handle, fault)

    def close(self):
        if self.handle:
            dms_stepper_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
