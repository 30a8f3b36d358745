"""Python binding of the C ABI in include/zo.h and include/zo_ops.h (ctypes).

Argument marshalling only: every step of the probe step runs in the CUDA
library ``libzo_b200.so`` built in-tree by ``zeroth_order_fine_b200.build``.
PyTorch provides device memory and the stream.  When the library is missing
the import of any entry point raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from . import workload as wl

_HERE = os.path.dirname(os.path.abspath(__file__))
# ZO_LIB=debug loads the debug build (device bounds checks, see zo_ops.h zo_debug_word)
LIB_PATH = os.path.join(_HERE, "libzo_b200_debug.so" if os.environ.get("ZO_LIB") == "debug"
                        else "libzo_b200.so")

ZO_OK, ZO_ERR_ARG, ZO_ERR_STATE, ZO_ERR_CUDA, ZO_ERR_OOM, ZO_ERR_NONFINITE, ZO_ERR_TIMEOUT, \
    ZO_ERR_UNSUPPORTED = range(8)
ERR_NAMES = {0: "ZO_OK", 1: "ZO_ERR_ARG", 2: "ZO_ERR_STATE", 3: "ZO_ERR_CUDA", 4: "ZO_ERR_OOM",
             5: "ZO_ERR_NONFINITE", 6: "ZO_ERR_TIMEOUT", 7: "ZO_ERR_UNSUPPORTED"}
IMPL_AUTO, IMPL_CUDA_CORES, IMPL_TENSOR_CORES = 0, 1, 2

c_void_p = ctypes.c_void_p
c_int32 = ctypes.c_int32
c_uint32 = ctypes.c_uint32
c_uint64 = ctypes.c_uint64


class ZoError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


class zo_model_desc(ctypes.Structure):
    _fields_ = [("arch", c_int32), ("n_layers", c_int32), ("d_model", c_int32),
                ("n_heads", c_int32), ("n_kv_heads", c_int32), ("head_dim", c_int32),
                ("d_ffn", c_int32), ("vocab", c_int32), ("max_pos", c_int32),
                ("norm_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("dtype", c_int32), ("tie_lm_head", c_int32)]


class zo_layer_weights(ctypes.Structure):
    _fields_ = [("w", c_void_p * 7), ("b", c_void_p * 7), ("ln1_w", c_void_p),
                ("ln1_b", c_void_p), ("ln2_w", c_void_p), ("ln2_b", c_void_p),
                ("q_norm", c_void_p), ("k_norm", c_void_p)]


class zo_weights(ctypes.Structure):
    _fields_ = [("tok_embed", c_void_p), ("pos_embed", c_void_p), ("final_w", c_void_p),
                ("final_b", c_void_p), ("lm_head", c_void_p),
                ("layers", ctypes.POINTER(zo_layer_weights))]


class zo_targets(ctypes.Structure):
    _fields_ = [("layer_mask_lo", c_uint64), ("layer_mask_hi", c_uint64),
                ("matrix_mask", c_uint32), ("scale_mode", c_int32)]


class zo_options(ctypes.Structure):
    _fields_ = [("run_seed", c_uint64), ("lazy_interval", c_int32), ("rank", c_int32),
                ("targets", zo_targets), ("max_tokens", c_int32), ("max_rows", c_int32),
                ("max_scored", c_int32), ("max_slots", c_int32), ("start_step", c_uint64),
                ("stream", c_void_p), ("impl", c_int32), ("profile", c_int32), ("fp8", c_int32),
                ("max_new", c_int32)]


class zo_stats_t(ctypes.Structure):
    _fields_ = [("steps", c_uint64), ("score_calls", c_uint64), ("tokens_scored", c_uint64),
                ("positions_scored", c_uint64), ("ms_plan", ctypes.c_double),
                ("ms_score", ctypes.c_double), ("ms_step", ctypes.c_double),
                ("state_transition_bytes", c_uint64), ("dense_ref_bytes", c_uint64),
                ("dense_ref_bytes_targets", c_uint64), ("bank_slots", c_int32),
                ("last_error_code", c_int32), ("kernel_launches", c_uint64),
                ("gemm_launches", c_uint64), ("gemm_ms", ctypes.c_double),
                ("gemm_flops", ctypes.c_double), ("tc_gemm_launches", c_uint64),
                ("tc_gemm_ms", ctypes.c_double), ("tc_gemm_flops", ctypes.c_double),
                ("cuda_core_gemm_launches", c_uint64), ("graph_captures", c_uint64),
                ("graph_replays", c_uint64)]


class zo_qk_norm_rope_args(ctypes.Structure):
    _fields_ = [("tok_pos", c_void_p), ("q_norm", c_void_p), ("k_norm", c_void_p),
                ("rope_cos", c_void_p), ("rope_sin", c_void_p), ("eps", ctypes.c_float),
                ("n_q_heads", c_int32), ("n_kv_heads", c_int32)]


_I32P = ctypes.POINTER(c_int32)
_F32P = ctypes.POINTER(ctypes.c_float)
_F64P = ctypes.POINTER(ctypes.c_double)

# name -> (restype, argtypes)
_SIGS = {
    "zo_create": (c_int32, [ctypes.POINTER(zo_model_desc), ctypes.POINTER(zo_weights),
                            ctypes.POINTER(zo_options), ctypes.POINTER(c_void_p)]),
    "zo_destroy": (None, [c_void_p]),
    "zo_last_error": (ctypes.c_char_p, [c_void_p]),
    "zo_op_last_error": (ctypes.c_char_p, []),
    "zo_debug_build": (ctypes.c_int, []),
    "zo_debug_word": (ctypes.c_uint32, [ctypes.c_int32]),
    "zo_probe_plan": (c_int32, [c_void_p, c_uint64, c_int32, ctypes.c_float,
                                ctypes.POINTER(zo_targets), ctypes.POINTER(c_void_p)]),
    "zo_score": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                           c_void_p, c_void_p]),
    "zo_score_cobatch": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p,
                                   c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_void_p,
                                   c_void_p, c_void_p]),
    "zo_score_foreground": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p]),
    "zo_generate": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_int32, c_void_p, c_void_p,
                              c_void_p, c_void_p]),
    "zo_step": (c_int32, [c_void_p, ctypes.c_float, c_void_p]),
    "zo_step_graph": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_void_p, ctypes.c_float,
                                ctypes.c_float, c_void_p, c_void_p]),
    "zo_objective_sums": (c_int32, [c_void_p, c_void_p]),
    "zo_step_from_sums": (c_int32, [c_void_p, ctypes.c_float, c_void_p, c_void_p]),
    "zo_stats": (c_int32, [c_void_p, ctypes.POINTER(zo_stats_t)]),
    "zo_save_state": (c_int32, [c_void_p, c_void_p, ctypes.POINTER(ctypes.c_size_t)]),
    "zo_load_state": (c_int32, [c_void_p, c_void_p, ctypes.c_size_t]),
    "zo_read_factors": (c_int32, [c_void_p, c_int32, c_int32, c_void_p, c_void_p]),
    "zo_read_bank": (c_int32, [c_void_p, c_int32, c_int32, c_int32, c_void_p]),
    "zo_init_tensor": (c_int32, [c_void_p, c_uint64, c_uint64, c_uint32, c_uint32,
                                 ctypes.c_float, ctypes.c_float, c_int32, c_void_p]),
    "zo_op_linear": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_int32,
                               c_int32, c_int32, c_int32, c_int32, c_void_p]),
    "zo_op_linear_decode": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                      c_int32, c_int32, c_int32, c_void_p, ctypes.c_size_t,
                                      c_void_p]),
    "zo_op_linear_ext": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int32,
                                   c_void_p, c_int32, c_int32, c_int32, c_int32, c_int32,
                                   ctypes.POINTER(zo_qk_norm_rope_args), c_void_p]),
    "zo_op_rope_table": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, ctypes.c_double,
                                   c_void_p]),
    "zo_op_set_wait_limit": (ctypes.c_int64, [ctypes.c_int64]),
    "zo_op_quantize_rows_e4m3": (c_int32, [c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                           c_void_p, c_void_p]),
    "zo_op_linear_fp8": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_int32, c_int32, c_int32, c_int32, c_void_p]),
    "zo_op_lm_head_workspace": (ctypes.c_size_t, [c_int32, c_int32, c_int32]),
    "zo_op_lm_head_logprob": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                        c_int32, c_void_p, c_void_p, ctypes.c_size_t, c_int32,
                                        c_void_p]),
    "zo_op_attention": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                  c_int32, c_int32, c_void_p, ctypes.c_size_t, c_int32, c_void_p]),
    "zo_op_error_word": (c_int32, []),
    "zo_op_lm_head_noalloc_capacity": (ctypes.c_size_t, []),
    "zo_op_lm_head_logprob_noalloc": (c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                                c_int32, c_int32, c_void_p, c_int32, c_void_p]),
}

EXPORTED = tuple(_SIGS)
_LIB: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The CUDA library; raises when it has not been built (no fallback exists)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m zeroth_order_fine_b200.build` (--debug for the debug "
                               "build; needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return int(t)


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(rc: int, handle=None) -> None:
    if rc != ZO_OK:
        msg = lib().zo_last_error(handle)
        raise ZoError(rc, msg.decode() if msg else "")


def _check_op(rc: int) -> None:
    if rc != ZO_OK:
        msg = lib().zo_op_last_error() if rc == ZO_ERR_CUDA else b""
        raise ZoError(rc, msg.decode() if msg else "")


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


# ---- model weights on the device --------------------------------------------------------

def torch_dtype(dtype: int):
    return torch.bfloat16 if dtype == wl.DTYPE_BF16 else torch.float32


def zo_init_tensor(t: torch.Tensor, weight_seed: int, layer: int, tensor: int, std: float,
                   mean: float, stream=None) -> None:
    dtype = wl.DTYPE_BF16 if t.dtype == torch.bfloat16 else wl.DTYPE_FP32
    _check(lib().zo_init_tensor(_ptr(t), t.numel(), weight_seed, layer, tensor, std, mean, dtype,
                                _stream(stream)))


class DeviceModel:
    """Random-init weights of a model shape, drawn on the device from the counter stream.

    Keeps the tensors alive and builds the zo_model_desc / zo_weights
    structures.  ``layers`` limits how many decoder layers are allocated
    (all by default).
    """

    def __init__(self, shape: wl.ModelShape, weight_seed: int = 0, device: str = "cuda"):
        self.shape = shape
        sh = shape
        dt = torch_dtype(sh.dtype)
        G = wl.GLOBAL_LAYER
        S = wl.INIT_STD
        self.tensors: List[torch.Tensor] = []

        def new(shape_, dtype, layer, tid, mean=0.0):
            t = torch.empty(shape_, dtype=dtype, device=device)
            zo_init_tensor(t, weight_seed, layer, tid, S, mean)
            self.tensors.append(t)
            return t

        d = sh.d_model
        self.tok_embed = new((sh.vocab, d), dt, G, wl.T_TOK_EMBED)
        self.pos_embed = new((sh.max_pos, d), dt, G, wl.T_POS_EMBED) if sh.arch == wl.ARCH_OPT else None
        self.final_w = new((d,), torch.float32, G, wl.T_FINAL_W, 1.0)
        self.final_b = new((d,), torch.float32, G, wl.T_FINAL_B) if sh.arch == wl.ARCH_OPT else None
        self.lm_head = None if sh.tie_lm_head else new((sh.vocab, d), dt, G, wl.T_LM_HEAD)
        self.layers: List[Dict[str, torch.Tensor]] = []
        for l in range(sh.n_layers):
            p: Dict[str, torch.Tensor] = {}
            for m in sh.matrices():
                di, do = sh.matrix_dims(m)
                p[f"W{m}"] = new((do, di), dt, l, m)
                if sh.arch == wl.ARCH_OPT:
                    p[f"b{m}"] = new((do,), torch.float32, l, wl.T_BIAS0 + m)
            p["ln1_w"] = new((d,), torch.float32, l, wl.T_LN1_W, 1.0)
            p["ln2_w"] = new((d,), torch.float32, l, wl.T_LN2_W, 1.0)
            if sh.arch == wl.ARCH_OPT:
                p["ln1_b"] = new((d,), torch.float32, l, wl.T_LN1_B)
                p["ln2_b"] = new((d,), torch.float32, l, wl.T_LN2_B)
            else:
                p["q_norm"] = new((sh.head_dim,), torch.float32, l, wl.T_QNORM, 1.0)
                p["k_norm"] = new((sh.head_dim,), torch.float32, l, wl.T_KNORM, 1.0)
            self.layers.append(p)

    def desc(self) -> zo_model_desc:
        sh = self.shape
        return zo_model_desc(sh.arch, sh.n_layers, sh.d_model, sh.n_heads, sh.n_kv_heads,
                             sh.head_dim, sh.d_ffn, sh.vocab, sh.max_pos, sh.norm_eps,
                             sh.rope_theta, sh.dtype, int(sh.tie_lm_head))

    def weights(self) -> zo_weights:
        arr = (zo_layer_weights * len(self.layers))()
        for i, p in enumerate(self.layers):
            lw = arr[i]
            for m in range(7):
                lw.w[m] = _ptr(p.get(f"W{m}"))
                lw.b[m] = _ptr(p.get(f"b{m}"))
            lw.ln1_w, lw.ln1_b = _ptr(p["ln1_w"]), _ptr(p.get("ln1_b"))
            lw.ln2_w, lw.ln2_b = _ptr(p["ln2_w"]), _ptr(p.get("ln2_b"))
            lw.q_norm, lw.k_norm = _ptr(p.get("q_norm")), _ptr(p.get("k_norm"))
        self._layer_arr = arr
        return zo_weights(_ptr(self.tok_embed), _ptr(self.pos_embed), _ptr(self.final_w),
                          _ptr(self.final_b), _ptr(self.lm_head),
                          ctypes.cast(arr, ctypes.POINTER(zo_layer_weights)))


def make_targets(n_layers: int, matrices: Sequence[int], scale_mode: int,
                 layers: Optional[Sequence[int]] = None) -> zo_targets:
    ls = range(n_layers) if layers is None else layers
    lo = hi = 0
    for l in ls:
        if l < 64:
            lo |= 1 << l
        else:
            hi |= 1 << (l - 64)
    mm = 0
    for m in matrices:
        mm |= 1 << m
    return zo_targets(lo, hi, mm, scale_mode)


# ---- the C-ABI calls ------------------------------------------------------------------

class Handle:
    """Owner of a zo_handle*: create / plan / score / step / state, one stream."""

    def __init__(self, model: DeviceModel, run_seed: int, nu: int, rank: int,
                 targets: zo_targets, max_tokens: int, max_rows: int, max_scored: int,
                 max_slots: int = 32, start_step: int = 0, stream=None, impl: int = 0,
                 profile: int = 0, fp8: int = 0, max_new: int = 0):
        self.model = model
        self.targets = targets
        self.rank = rank
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self._desc = model.desc()
        self._w = model.weights()
        opt = zo_options(run_seed, nu, rank, targets, max_tokens, max_rows, max_scored, max_slots,
                         start_step, _stream(self.stream), impl, profile, fp8, max_new)
        h = c_void_p()
        rc = lib().zo_create(ctypes.byref(self._desc), ctypes.byref(self._w), ctypes.byref(opt),
                             ctypes.byref(h))
        _check(rc, None)
        self.h = h
        self.plan = None

    def close(self):
        if getattr(self, "h", None):
            lib().zo_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # zo_probe_plan
    def zo_probe_plan(self, step: int, eps: float):
        p = c_void_p()
        _check(lib().zo_probe_plan(self.h, step, self.rank, eps, ctypes.byref(self.targets),
                                   ctypes.byref(p)), self.h)
        self.plan = p
        return p

    # zo_score
    def zo_score(self, tokens: torch.Tensor, seq_lens, target_lens,
                 target_ids: Optional[torch.Tensor] = None, want_logprob: bool = False):
        sl, tl = _i32(seq_lens), _i32(target_lens)
        B = len(sl)
        _cuda_args({"tokens": (int(sl.sum()),), "target_ids": (int(tl.sum()),)},
                   {"tokens": (torch.int32,), "target_ids": (torch.int32,)},
                   tokens=tokens, target_ids=target_ids)
        dev = tokens.device
        Lp = torch.empty(B, dtype=torch.float32, device=dev)
        Lm = torch.empty(B, dtype=torch.float32, device=dev)
        lp = torch.empty(2 * int(tl.sum()), dtype=torch.float32, device=dev) if want_logprob else None
        _check(lib().zo_score(self.plan, _ptr(tokens), B, _ptr(sl), _ptr(tl), _ptr(target_ids),
                              _ptr(Lp), _ptr(Lm), _ptr(lp)), self.h)
        return Lp, Lm, lp

    # zo_score_cobatch
    def zo_score_cobatch(self, tokens, seq_lens, target_lens, fg_tokens, fg_seq_lens,
                         fg_target_lens, want_logprob: bool = False):
        sl, tl = _i32(seq_lens), _i32(target_lens)
        fsl, ftl = _i32(fg_seq_lens), _i32(fg_target_lens)
        B, F = len(sl), len(fsl)
        _cuda_args({"tokens": (int(sl.sum()),), "fg_tokens": (int(fsl.sum()),)},
                   {"tokens": (torch.int32,), "fg_tokens": (torch.int32,)},
                   tokens=tokens, fg_tokens=fg_tokens)
        dev = tokens.device
        Lp = torch.empty(B, dtype=torch.float32, device=dev)
        Lm = torch.empty(B, dtype=torch.float32, device=dev)
        lp = torch.empty(2 * int(tl.sum()), dtype=torch.float32, device=dev) if want_logprob else None
        flp = torch.empty(int(ftl.sum()), dtype=torch.float32, device=dev)
        _check(lib().zo_score_cobatch(self.plan, _ptr(tokens), B, _ptr(sl), _ptr(tl), None,
                                      _ptr(Lp), _ptr(Lm), _ptr(lp), _ptr(fg_tokens), F,
                                      _ptr(fsl), _ptr(ftl), _ptr(flp)), self.h)
        return Lp, Lm, lp, flp

    # zo_generate: greedy generation queries of both candidates
    def zo_generate(self, tokens, seq_lens, n_new: int):
        sl = _i32(seq_lens)
        B = len(sl)
        _cuda_args({"tokens": (int(sl.sum()),)}, {"tokens": (torch.int32,)}, tokens=tokens)
        dev = tokens.device
        Lp = torch.empty(B, dtype=torch.float32, device=dev)
        Lm = torch.empty(B, dtype=torch.float32, device=dev)
        gt = torch.empty(2 * B, n_new, dtype=torch.int32, device=dev)
        gl = torch.empty(2 * B, n_new, dtype=torch.float32, device=dev)
        _check(lib().zo_generate(self.plan, _ptr(tokens), B, _ptr(sl), n_new, _ptr(gt), _ptr(gl),
                                 _ptr(Lp), _ptr(Lm)), self.h)
        return Lp, Lm, gt, gl

    # zo_score_foreground
    def zo_score_foreground(self, fg_tokens, fg_seq_lens, fg_target_lens):
        fsl, ftl = _i32(fg_seq_lens), _i32(fg_target_lens)
        _cuda_args({"fg_tokens": (int(fsl.sum()),)}, {"fg_tokens": (torch.int32,)},
                   fg_tokens=fg_tokens)
        flp = torch.empty(int(ftl.sum()), dtype=torch.float32, device=fg_tokens.device)
        _check(lib().zo_score_foreground(self.h, _ptr(fg_tokens), len(fsl), _ptr(fsl), _ptr(ftl),
                                         _ptr(flp)), self.h)
        return flp

    # zo_step
    def zo_step(self, lr: float, want_c: bool = True) -> Optional[float]:
        c = ctypes.c_double(0.0)
        _check(lib().zo_step(self.h, lr, ctypes.byref(c) if want_c else None), self.h)
        return c.value if want_c else None

    # zo_step_graph: the library bakes the output pointers into its graph, so the
    # handle keeps one pair of L+/L- buffers per batch size; the returned tensors are
    # overwritten by the next step of the same size
    def zo_step_graph(self, tokens, seq_lens, target_lens, eps: float, lr: float):
        sl, tl = _i32(seq_lens), _i32(target_lens)
        B = len(sl)
        _cuda_args({"tokens": (int(sl.sum()),)}, {"tokens": (torch.int32,)}, tokens=tokens)
        bufs = self.__dict__.setdefault("_graph_out", {})
        if B not in bufs:
            bufs[B] = (torch.empty(B, dtype=torch.float32, device=tokens.device),
                       torch.empty(B, dtype=torch.float32, device=tokens.device))
        Lp, Lm = bufs[B]
        _check(lib().zo_step_graph(self.h, _ptr(tokens), B, _ptr(sl), _ptr(tl), eps, lr,
                                   _ptr(Lp), _ptr(Lm)), self.h)
        return Lp, Lm

    def zo_objective_sums(self, dev_sums: torch.Tensor) -> None:
        _cuda_args({"dev_sums": (2,)}, {"dev_sums": (torch.float64,)}, dev_sums=dev_sums)
        _check(lib().zo_objective_sums(self.h, _ptr(dev_sums)), self.h)

    def zo_step_from_sums(self, lr: float, dev_sums: torch.Tensor, want_c: bool = True):
        _cuda_args({"dev_sums": (2,)}, {"dev_sums": (torch.float64,)}, dev_sums=dev_sums)
        c = ctypes.c_double(0.0)
        _check(lib().zo_step_from_sums(self.h, lr, _ptr(dev_sums),
                                       ctypes.byref(c) if want_c else None), self.h)
        return c.value if want_c else None

    def zo_stats(self) -> Dict[str, float]:
        s = zo_stats_t()
        _check(lib().zo_stats(self.h, ctypes.byref(s)), self.h)
        return {f: getattr(s, f) for f, _ in zo_stats_t._fields_}

    def zo_save_state(self) -> bytes:
        n = ctypes.c_size_t(0)
        _check(lib().zo_save_state(self.h, None, ctypes.byref(n)), self.h)
        buf = ctypes.create_string_buffer(n.value)
        _check(lib().zo_save_state(self.h, buf, ctypes.byref(n)), self.h)
        return buf.raw[: n.value]

    def zo_load_state(self, data: bytes) -> None:
        buf = ctypes.create_string_buffer(data, len(data))
        _check(lib().zo_load_state(self.h, buf, len(data)), self.h)

    def zo_read_factors(self, layer: int, matrix: int):
        di, do = self.model.shape.matrix_dims(matrix)
        U = np.empty((di, self.rank), dtype=np.float32)
        V = np.empty((do, self.rank), dtype=np.float32)
        _check(lib().zo_read_factors(self.plan, layer, matrix, _ptr(U), _ptr(V)), self.h)
        return U, V

    def zo_read_bank(self, layer: int, matrix: int, slot: int) -> np.ndarray:
        di, _ = self.model.shape.matrix_dims(matrix)
        A = np.empty((di, self.rank), dtype=np.float32)
        _check(lib().zo_read_bank(self.h, layer, matrix, slot, _ptr(A)), self.h)
        return A


# ---- kernel-level ops -----------------------------------------------------------------

def _cuda_args(shapes: dict, dtypes: dict = None, **tensors) -> None:
    """The library takes raw device pointers: every tensor it reads or writes must be a
    contiguous CUDA tensor on one device, with the shape (a tuple, None entries free) and
    dtype the op expects; a wrong one raises here instead of reaching a kernel."""
    dev = None
    dtypes = dtypes or {}
    for name, t in tensors.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other arguments on {dev}")
        want = shapes.get(name)
        if want is not None and (t.dim() != len(want) or
                                 any(w is not None and w != n for w, n in zip(want, t.shape))):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want}")
        if name in dtypes and t.dtype not in dtypes[name]:
            raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes[name]}")


_FLOATS = (torch.float32, torch.bfloat16)


def zo_op_linear(x: torch.Tensor, W: torch.Tensor, bias: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, act: int = 0, accumulate: bool = False,
                 impl: int = IMPL_AUTO) -> torch.Tensor:
    M, K = x.shape
    N = W.shape[0]
    dtype = wl.DTYPE_BF16 if x.dtype == torch.bfloat16 else wl.DTYPE_FP32
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32 if accumulate else x.dtype, device=x.device)
    _cuda_args({"W": (N, K), "bias": (N,), "out": (M, N)},
               {"x": _FLOATS, "W": (x.dtype,), "bias": (torch.float32,),
                "out": (torch.float32,) if accumulate else (x.dtype,)}, x=x, W=W, bias=bias, out=out)
    _check_op(lib().zo_op_linear(_ptr(x), _ptr(W), _ptr(bias), _ptr(out), M, N, K, dtype, act,
                              int(accumulate), impl, _stream()))
    return out


def zo_op_linear_decode(x: torch.Tensor, W: torch.Tensor, bias: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, act: int = 0, accumulate: bool = False,
                        ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The decode-step linear (bf16): split-K tensor-core GEMM through an fp32 workspace."""
    M, K = x.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32 if accumulate else x.dtype, device=x.device)
    if ws is None:
        ws = torch.empty(max(1, 16 * M * N), dtype=torch.float32, device=x.device)
    _cuda_args({"W": (N, K), "bias": (N,), "out": (M, N)},
               {"x": (torch.bfloat16,), "W": (torch.bfloat16,), "bias": (torch.float32,),
                "out": (torch.float32,) if accumulate else (torch.bfloat16,), "ws": (torch.float32,)},
               x=x, W=W, bias=bias, out=out, ws=ws)
    _check_op(lib().zo_op_linear_decode(_ptr(x), _ptr(W), _ptr(bias), _ptr(out), M, N, K, act,
                                     int(accumulate), _ptr(ws), ws.numel(), _stream()))
    return out


EPI_STORE, EPI_RELU, EPI_RESID, EPI_SWIGLU, EPI_QK_NORM_ROPE = 0, 1, 2, 5, 6


def zo_op_linear_ext(x: torch.Tensor, W: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     x2: Optional[torch.Tensor] = None, W2: Optional[torch.Tensor] = None,
                     epi: int = EPI_STORE, out: Optional[torch.Tensor] = None,
                     qk: Optional[dict] = None) -> torch.Tensor:
    """The perturbed linear of one fused group on the tensor cores (bf16): x W^T + x2 W2^T
    + b with the group's epilogue (store, ReLU, residual add, SwiGLU, q/k norm + RoPE).
    ``qk`` holds the ZO_EPI_QK_NORM_ROPE arguments: tok_pos, q_norm, k_norm, rope_cos,
    rope_sin (device tensors), eps, n_q_heads, n_kv_heads."""
    M, K = x.shape
    N = W.shape[0]
    K2 = 0 if x2 is None else x2.shape[1]
    if out is None:
        cols = N // 2 if epi == EPI_SWIGLU else N
        out = torch.empty(M, cols, dtype=torch.float32 if epi == EPI_RESID else torch.bfloat16,
                          device=x.device)
    _cuda_args({"W": (N, K), "bias": (N,), "x2": (M, K2), "W2": (N, K2)},
               {"x": (torch.bfloat16,), "W": (torch.bfloat16,), "bias": (torch.float32,),
                "x2": (torch.bfloat16,), "W2": (torch.bfloat16,)},
               x=x, W=W, bias=bias, x2=x2, W2=W2)
    if out.device != x.device or not out.is_cuda or out.stride(1) != 1 or out.shape[0] != M:
        raise ValueError("out must be a CUDA tensor with unit column stride and M rows")
    if out.dtype != (torch.float32 if epi == EPI_RESID else torch.bfloat16):
        raise ValueError("out must be float32 for the residual epilogue, else bfloat16")
    args = None
    if qk is not None:
        _cuda_args({}, {"tok_pos": (torch.int32,)}, tok_pos=qk["tok_pos"], q_norm=qk["q_norm"],
                   k_norm=qk["k_norm"], rope_cos=qk["rope_cos"], rope_sin=qk["rope_sin"], x=x)
        args = zo_qk_norm_rope_args(_ptr(qk["tok_pos"]), _ptr(qk["q_norm"]), _ptr(qk["k_norm"]),
                                    _ptr(qk["rope_cos"]), _ptr(qk["rope_sin"]), qk["eps"],
                                    qk["n_q_heads"], qk["n_kv_heads"])
    _check_op(lib().zo_op_linear_ext(_ptr(x), _ptr(W), _ptr(bias), _ptr(x2), _ptr(W2), K2, _ptr(out),
                                  out.stride(0), M, N, K, epi,
                                  ctypes.byref(args) if args is not None else None, _stream()))
    return out


def zo_op_rope_table(max_pos: int, head_dim: int, theta: float, device="cuda"):
    """(cos, sin) rotary tables [max_pos x head_dim/2] as zo_create builds them."""
    c = torch.empty(max_pos, head_dim // 2, dtype=torch.float32, device=device)
    s = torch.empty(max_pos, head_dim // 2, dtype=torch.float32, device=device)
    _check_op(lib().zo_op_rope_table(_ptr(c), _ptr(s), max_pos, head_dim, theta, _stream()))
    return c, s


def zo_op_set_wait_limit(cycles: int) -> int:
    """Bound of every mbarrier wait in the tensor-core GEMMs (<= 0: the default); returns
    the previous bound."""
    return int(lib().zo_op_set_wait_limit(cycles))


def zo_op_quantize_rows_e4m3(x: torch.Tensor):
    """(codes uint8 [rows, cols], scale float [rows]) of the E4M3 row quantiser."""
    rows, cols = x.shape
    dtype = wl.DTYPE_BF16 if x.dtype == torch.bfloat16 else wl.DTYPE_FP32
    _cuda_args({}, {"x": _FLOATS}, x=x)
    q = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    sc = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check_op(lib().zo_op_quantize_rows_e4m3(_ptr(x), dtype, rows, cols, _ptr(q), _ptr(sc),
                                          _stream()))
    return q, sc


def zo_op_linear_fp8(xq: torch.Tensor, sx: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                     bias: Optional[torch.Tensor] = None, act: int = 0) -> torch.Tensor:
    M, K = xq.shape
    N = wq.shape[0]
    _cuda_args({"sx": (M,), "wq": (N, K), "sw": (N,), "bias": (N,)},
               {"xq": (torch.uint8,), "wq": (torch.uint8,), "sx": (torch.float32,),
                "sw": (torch.float32,), "bias": (torch.float32,)},
               xq=xq, sx=sx, wq=wq, sw=sw, bias=bias)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=xq.device)
    _check_op(lib().zo_op_linear_fp8(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(bias), _ptr(y),
                                  M, N, K, act, _stream()))
    return y


def zo_op_lm_head_logprob(h: torch.Tensor, E: torch.Tensor, targets: torch.Tensor,
                          impl: int = IMPL_AUTO) -> torch.Tensor:
    S, d = h.shape
    V = E.shape[0]
    _cuda_args({"E": (V, d), "targets": (S,)},
               {"h": _FLOATS, "E": (h.dtype,), "targets": (torch.int32,)}, h=h, E=E, targets=targets)
    dtype = wl.DTYPE_BF16 if h.dtype == torch.bfloat16 else wl.DTYPE_FP32
    ws_bytes = lib().zo_op_lm_head_workspace(S, V, impl)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=h.device)
    out = torch.empty(S, dtype=torch.float32, device=h.device)
    _check_op(lib().zo_op_lm_head_logprob(_ptr(h), _ptr(E), _ptr(targets), S, V, d, dtype, _ptr(out),
                                       _ptr(ws), ws.numel(), impl, _stream()))
    return out


def zo_op_attention(qkv: torch.Tensor, seq_lens, n_heads: int, n_kv_heads: int,
                    head_dim: int, impl: int = IMPL_AUTO,
                    out: Optional[torch.Tensor] = None) -> torch.Tensor:
    sl = _i32(seq_lens)
    T = qkv.shape[0]
    _cuda_args({"qkv": (int(sl.sum()), (n_heads + 2 * n_kv_heads) * head_dim)}, {"qkv": _FLOATS},
               qkv=qkv)
    dtype = wl.DTYPE_BF16 if qkv.dtype == torch.bfloat16 else wl.DTYPE_FP32
    if out is None:
        out = torch.empty(T, n_heads * head_dim, dtype=qkv.dtype, device=qkv.device)
    elif (out.shape != (T, n_heads * head_dim) or out.dtype != qkv.dtype or not out.is_cuda
          or not out.is_contiguous()):
        raise ValueError("out must be a contiguous CUDA tensor [T x n_heads*head_dim] of qkv's dtype")
    ws = torch.empty(4 * (2 * len(sl) + 2 + T // 64 + 1) + 256, dtype=torch.uint8, device=qkv.device)
    _check_op(lib().zo_op_attention(_ptr(qkv), _ptr(out), _ptr(sl), len(sl), n_heads, n_kv_heads,
                                 head_dim, dtype, _ptr(ws), ws.numel(), impl, _stream()))
    return out


def zo_op_lm_head_logprob_noalloc(h: torch.Tensor, E: torch.Tensor, targets: torch.Tensor,
                                   out: torch.Tensor, impl: int = IMPL_AUTO) -> torch.Tensor:
    """The lm_head log-probabilities with the library's own fixed scratch (no
    workspace, no allocation inside the call); ``out`` is the caller's buffer."""
    S, d = h.shape
    for name, t in (("h", h), ("E", E), ("targets", targets), ("out", out)):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if t.device != h.device:
            raise ValueError(f"{name} is on {t.device}, h on {h.device}")
    if E.dtype != h.dtype or E.dim() != 2 or E.shape[1] != d:
        raise ValueError("E must be [vocab x d] in h's dtype")
    if targets.dtype != torch.int32 or targets.numel() != S:
        raise ValueError("targets must be int32 with one entry per row of h")
    if out.dtype != torch.float32 or out.numel() < S:
        raise ValueError("out must be float32 with room for one value per row of h")
    dtype = wl.DTYPE_BF16 if h.dtype == torch.bfloat16 else wl.DTYPE_FP32
    _check_op(lib().zo_op_lm_head_logprob_noalloc(_ptr(h), _ptr(E), _ptr(targets), S, E.shape[0], d,
                                               dtype, _ptr(out), impl, _stream()))
    return out


def zo_op_error_word() -> int:
    return int(lib().zo_op_error_word())
