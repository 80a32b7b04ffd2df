"""Thin ctypes binding over the C ABI in ``include/spec_verify.h``.

Argument marshalling only: every step of verification runs in the CUDA
kernels of ``lib/libspecverify.so``.  Torch supplies device memory and the
current stream.  There is no fallback: if the library is missing or the
tensors are not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libspecverify.so")

SV_OK = 0
SV_DTYPE_F32, SV_DTYPE_BF16 = 0, 1
ROW_BAD_TOKEN, ROW_BAD_LOGITS, ROW_BAD_TEMPERATURE, ROW_RESIDUAL_ZERO, ROW_BAD_UNIFORM = 1, 2, 4, 8, 16
EXPORTED = ("spec_verify", "spec_verify_workspace_size", "spec_verify_workspace_init",
            "spec_verify_status_string", "spec_verify_kernels_per_call", "spec_verify_noalloc",
            "spec_verify_fanout", "spec_verify_topf", "spec_verify_cache_lookup",
            "spec_verify_bandit_state_size", "spec_verify_bandit_init", "spec_verify_bandit_step",
            "spec_verify_bandit_simulate", "spec_verify_tree", "spec_verify_tree_prune",
            "spec_verify_lowrank_workspace_size", "spec_verify_lowrank_down", "spec_verify_lowrank_up",
            "spec_verify_lowrank_head")
MAX_TOPF = 32
MAX_ARMS = 16
BANDIT_UCB1, BANDIT_THOMPSON, BANDIT_THOMPSON_BETA = 0, 1, 2
MAX_TREE_NODES = 64
ROW_BAD_TREE = 32

_lib = None


class SpecVerifyError(ValueError):
    """A non-OK status returned by the C ABI."""

    def __init__(self, status: int, message: str):
        super().__init__(f"spec_verify status {status}: {message}")
        self.status = status


def load_library(path: str = LIB_PATH):
    """Load the C-ABI library and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.spec_verify_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.spec_verify_workspace_size.restype = sz
    lib.spec_verify_workspace_init.argtypes = [vp, sz, vp]
    lib.spec_verify_workspace_init.restype = i32
    lib.spec_verify.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, sz, vp, vp, vp]
    lib.spec_verify.restype = i32
    lib.spec_verify_kernels_per_call.argtypes = [i32, i32, i32, i32]
    lib.spec_verify_kernels_per_call.restype = i32
    lib.spec_verify_status_string.argtypes = [i32]
    lib.spec_verify_status_string.restype = ctypes.c_char_p
    lib.spec_verify_fanout.argtypes = [ctypes.c_double, i32, i32, vp]
    lib.spec_verify_fanout.restype = i32
    lib.spec_verify_topf.argtypes = [vp, vp, i32, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp]
    lib.spec_verify_topf.restype = i32
    lib.spec_verify_cache_lookup.argtypes = [vp, vp, vp, vp, i32, i32, vp, vp]
    lib.spec_verify_cache_lookup.restype = i32
    lib.spec_verify_bandit_state_size.argtypes = [i32]
    lib.spec_verify_bandit_state_size.restype = sz
    lib.spec_verify_bandit_init.argtypes = [vp, i32, vp]
    lib.spec_verify_bandit_init.restype = i32
    lib.spec_verify_bandit_step.argtypes = [vp, i32, i32, i32, vp, vp, vp, i32, vp, vp]
    lib.spec_verify_bandit_step.restype = i32
    lib.spec_verify_bandit_simulate.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
    lib.spec_verify_bandit_simulate.restype = i32
    lib.spec_verify_tree.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.spec_verify_tree.restype = i32
    lib.spec_verify_tree_prune.argtypes = [vp, i32, vp, vp, vp, ctypes.c_double, i32, i32, i32, vp, vp, vp]
    lib.spec_verify_tree_prune.restype = i32
    lib.spec_verify_lowrank_workspace_size.argtypes = [i32, i32, i32]
    lib.spec_verify_lowrank_workspace_size.restype = sz
    lib.spec_verify_lowrank_down.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
    lib.spec_verify_lowrank_down.restype = i32
    lib.spec_verify_lowrank_up.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp]
    lib.spec_verify_lowrank_up.restype = i32
    lib.spec_verify_lowrank_head.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp]
    lib.spec_verify_lowrank_head.restype = i32
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().spec_verify_status_string(int(status)).decode()


def _dt_code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return SV_DTYPE_F32
    if dtype == torch.bfloat16:
        return SV_DTYPE_BF16
    raise TypeError(f"logits dtype must be float32 or bfloat16, got {dtype}")


def workspace_size(B: int, gamma: int, V: int, dtype: torch.dtype) -> int:
    return int(load_library().spec_verify_workspace_size(B, gamma, V, _dt_code(dtype)))


def kernels_per_call(B: int, gamma: int, V: int, dtype: torch.dtype) -> int:
    return int(load_library().spec_verify_kernels_per_call(B, gamma, V, _dt_code(dtype)))


_ws_cache: Dict[Tuple, torch.Tensor] = {}


def workspace_for(B: int, gamma: int, V: int, dtype: torch.dtype, device) -> torch.Tensor:
    """A workspace cached per (device, shape); it needs no initialisation.  Calls
    that share it must be ordered on one stream; pass ``workspace=`` to run shapes
    concurrently."""
    device = torch.device(device)
    key = (device.index, B, gamma, V, dtype)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(max(1, workspace_size(B, gamma, V, dtype)), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _check(t: torch.Tensor, name: str, dtype, shape, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def verify(target: torch.Tensor, draft: torch.Tensor, draft_tokens: torch.Tensor,
           temperature: torch.Tensor, u_accept: torch.Tensor, u_resample: torch.Tensor, *,
           return_log_norm: bool = False, return_row_status: bool = False,
           out_tokens: torch.Tensor | None = None, out_n_accepted: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None):
    """Verify B sequences on the GPU (see include/spec_verify.h for the rule).

    target [B, gamma+1, V] and draft [B, gamma, V] (float32 or bfloat16),
    draft_tokens [B, gamma] int32, temperature [B] float32 (0 = greedy),
    u_accept [B, gamma] and u_resample [B] float32 in (0, 1), all on one CUDA device.
    Returns (out_tokens [B, gamma+1] int32, n_accepted [B] int32) plus, if asked,
    log_norm [B, 2*gamma+1] float64 and row_status [B] int32.  Runs asynchronously on
    the current stream (or ``stream``); raises SpecVerifyError on a non-OK status."""
    lib = load_library()
    if not isinstance(target, torch.Tensor) or target.device.type != "cuda":
        raise ValueError("target must be a CUDA tensor")
    device = target.device
    if target.dim() != 3:
        raise ValueError("target must be [B, gamma+1, V]")
    B, g1, V = target.shape
    gamma = g1 - 1
    dt = _dt_code(target.dtype)
    _check(target, "target", None, (B, gamma + 1, V), device)
    _check(draft, "draft", target.dtype, (B, gamma, V), device)
    _check(draft_tokens, "draft_tokens", torch.int32, (B, gamma), device)
    _check(temperature, "temperature", torch.float32, (B,), device)
    _check(u_accept, "u_accept", torch.float32, (B, gamma), device)
    _check(u_resample, "u_resample", torch.float32, (B,), device)
    if out_tokens is None:
        out_tokens = torch.empty((B, gamma + 1), dtype=torch.int32, device=device)
    if out_n_accepted is None:
        out_n_accepted = torch.empty((B,), dtype=torch.int32, device=device)
    _check(out_tokens, "out_tokens", torch.int32, (B, gamma + 1), device)
    _check(out_n_accepted, "out_n_accepted", torch.int32, (B,), device)
    log_norm = torch.empty((B, 2 * gamma + 1), dtype=torch.float64, device=device) if return_log_norm else None
    row_status = torch.empty((B,), dtype=torch.int32, device=device) if return_row_status else None
    if workspace is None:
        workspace = workspace_for(B, gamma, V, target.dtype, device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        st = lib.spec_verify(target.data_ptr(), draft.data_ptr(), dt, draft_tokens.data_ptr(),
                             temperature.data_ptr(), u_accept.data_ptr(), u_resample.data_ptr(),
                             out_tokens.data_ptr(), out_n_accepted.data_ptr(), B, gamma, V,
                             workspace.data_ptr(), workspace.numel(),
                             log_norm.data_ptr() if log_norm is not None else None,
                             row_status.data_ptr() if row_status is not None else None,
                             s.cuda_stream)
    if st != SV_OK:
        raise SpecVerifyError(st, status_string(st))
    out = [out_tokens, out_n_accepted]
    if return_log_norm:
        out.append(log_norm)
    if return_row_status:
        out.append(row_status)
    return tuple(out)


def fanout(alpha: float, gamma: int, budget: int):
    """Cache slots per outcome n in [0, gamma] (host int32 array): geometric in n
    with acceptance rate alpha, summing to the budget."""
    import numpy as np
    F = np.empty((gamma + 1,), dtype=np.int32)
    st = load_library().spec_verify_fanout(float(alpha), int(gamma), int(budget), F.ctypes.data)
    if st != SV_OK:
        raise SpecVerifyError(st, status_string(st))
    return F


def _host_fanout(F, gamma):
    import numpy as np
    F = np.ascontiguousarray(F, dtype=np.int32).reshape(gamma + 1)
    return F, int(F.sum())


def topf(target: torch.Tensor, draft: torch.Tensor, temperature: torch.Tensor, log_norm: torch.Tensor,
         row_status: torch.Tensor, F, *, stream: torch.cuda.Stream | None = None):
    """Top-F_n tokens of the extra token's distribution for every outcome n, from
    spec_verify's log_norm and row_status: (tokens [B, sum F] int32, prob [B, sum F]
    float32) on the device."""
    lib = load_library()
    device = target.device
    B, g1, V = target.shape
    gamma = g1 - 1
    dt = _dt_code(target.dtype)
    _check(target, "target", None, (B, gamma + 1, V), device)
    _check(draft, "draft", target.dtype, (B, gamma, V), device)
    _check(temperature, "temperature", torch.float32, (B,), device)
    _check(log_norm, "log_norm", torch.float64, (B, 2 * gamma + 1), device)
    _check(row_status, "row_status", torch.int32, (B,), device)
    Fh, Ft = _host_fanout(F, gamma)
    tok = torch.empty((B, Ft), dtype=torch.int32, device=device)
    prob = torch.empty((B, Ft), dtype=torch.float32, device=device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        st = lib.spec_verify_topf(target.data_ptr(), draft.data_ptr(), dt, temperature.data_ptr(),
                                  log_norm.data_ptr(), row_status.data_ptr(), Fh.ctypes.data, B, gamma, V,
                                  tok.data_ptr(), prob.data_ptr(), s.cuda_stream)
    if st != SV_OK:
        raise SpecVerifyError(st, status_string(st))
    return tok, prob


def cache_lookup(out_tokens: torch.Tensor, n_accepted: torch.Tensor, cache_tokens: torch.Tensor, F, *,
                 stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Slot of each sequence's outcome (n, extra token) in its cache, else -1 ([B] int32)."""
    lib = load_library()
    device = out_tokens.device
    B, g1 = out_tokens.shape
    gamma = g1 - 1
    Fh, Ft = _host_fanout(F, gamma)
    _check(out_tokens, "out_tokens", torch.int32, (B, gamma + 1), device)
    _check(n_accepted, "n_accepted", torch.int32, (B,), device)
    _check(cache_tokens, "cache_tokens", torch.int32, (B, Ft), device)
    slot = torch.empty((B,), dtype=torch.int32, device=device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        st = lib.spec_verify_cache_lookup(out_tokens.data_ptr(), n_accepted.data_ptr(), cache_tokens.data_ptr(),
                                          Fh.ctypes.data, B, gamma, slot.data_ptr(), s.cuda_stream)
    if st != SV_OK:
        raise SpecVerifyError(st, status_string(st))
    return slot


def _raise_if(st: int):
    if st != SV_OK:
        raise SpecVerifyError(st, status_string(st))


def bandit_state(K: int, device="cuda", stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """A new bandit state on ``device`` ([2 + 2K] float64: t, arm, N, R), set to
    the empty state by the library on ``stream``."""
    lib = load_library()
    nbytes = lib.spec_verify_bandit_state_size(int(K))
    if nbytes == 0:
        raise SpecVerifyError(1, f"K must be in [1, {MAX_ARMS}]")
    device = torch.device(device)
    state = torch.empty((nbytes // 8,), dtype=torch.float64, device=device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_bandit_init(state.data_ptr(), int(K), s.cuda_stream))
    return state


def bandit_step(n_accepted: torch.Tensor, gamma: int, state: torch.Tensor, policy: int = BANDIT_UCB1,
                u1: torch.Tensor | None = None, u2: torch.Tensor | None = None,
                out_arm: torch.Tensor | None = None, *, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Reward the arm chosen last with the batch's accepted fraction and choose the
    next arm, on the device; returns ``out_arm`` ([1] int32, device)."""
    lib = load_library()
    device = state.device
    K = (state.numel() - 2) // 2
    _check(state, "state", torch.float64, (2 + 2 * K,), device)
    B = n_accepted.numel()
    _check(n_accepted, "n_accepted", torch.int32, (B,), device)
    for name, u in (("u1", u1), ("u2", u2)):
        if u is not None:
            _check(u, name, torch.float32, (K,), device)
    if out_arm is None:
        out_arm = torch.empty((1,), dtype=torch.int32, device=device)
    _check(out_arm, "out_arm", torch.int32, (1,), device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_bandit_step(n_accepted.data_ptr(), B, int(gamma), int(policy),
                                              u1.data_ptr() if u1 is not None else None,
                                              u2.data_ptr() if u2 is not None else None,
                                              state.data_ptr(), K, out_arm.data_ptr(), s.cuda_stream))
    return out_arm


def bandit_simulate(mu: torch.Tensor, T: int, policy: int, uniforms: torch.Tensor, *, with_state: bool = False,
                    stream: torch.cuda.Stream | None = None):
    """Regret of each run of the simulation ([runs] float64, device); with
    ``with_state`` also each run's final state ([runs][2 + 2K])."""
    lib = load_library()
    device = mu.device
    K = mu.numel()
    _check(mu, "mu", torch.float64, (K,), device)
    runs = uniforms.shape[0] if uniforms.dim() == 3 else -1
    _check(uniforms, "uniforms", torch.float32, (runs, int(T) + 1, 2 * K + 1), device)
    regret = torch.empty((runs,), dtype=torch.float64, device=device)
    state = torch.empty((runs, 2 + 2 * K), dtype=torch.float64, device=device) if with_state else None
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_bandit_simulate(mu.data_ptr(), K, int(T), int(policy), runs, uniforms.data_ptr(),
                                                  regret.data_ptr(), state.data_ptr() if with_state else None,
                                                  s.cuda_stream))
    return (regret, state) if with_state else regret


def tree_verify(target: torch.Tensor, draft: torch.Tensor, parent: torch.Tensor, tokens: torch.Tensor,
                temperature: torch.Tensor, u_accept: torch.Tensor, u_resample: torch.Tensor,
                keep: torch.Tensor | None = None, *, return_log_norm: bool = False, return_row_status: bool = False,
                stream: torch.cuda.Stream | None = None):
    """Verify B token trees on the GPU (see include/spec_verify.h).

    target, draft [B, N, V] (float32 or bfloat16); parent, tokens, u_accept [B, N];
    keep [B, N] int32 or None; temperature, u_resample [B].  Returns (out_nodes [B, N],
    out_tokens [B, N], n_accepted [B]) plus, if asked, log_norm [B, 2N] and row_status [B]."""
    lib = load_library()
    if not isinstance(target, torch.Tensor) or target.device.type != "cuda" or target.dim() != 3:
        raise ValueError("target must be a [B, N, V] CUDA tensor")
    device = target.device
    B, N, V = target.shape
    dt = _dt_code(target.dtype)
    _check(target, "target", None, (B, N, V), device)
    _check(draft, "draft", target.dtype, (B, N, V), device)
    for name, t in (("parent", parent), ("tokens", tokens)):
        _check(t, name, torch.int32, (B, N), device)
    if keep is not None:
        _check(keep, "keep", torch.int32, (B, N), device)
    _check(temperature, "temperature", torch.float32, (B,), device)
    _check(u_accept, "u_accept", torch.float32, (B, N), device)
    _check(u_resample, "u_resample", torch.float32, (B,), device)
    nodes = torch.empty((B, N), dtype=torch.int32, device=device)
    toks = torch.empty((B, N), dtype=torch.int32, device=device)
    n = torch.empty((B,), dtype=torch.int32, device=device)
    log_norm = torch.empty((B, 2 * N), dtype=torch.float64, device=device) if return_log_norm else None
    status = torch.empty((B,), dtype=torch.int32, device=device) if return_row_status else None
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_tree(target.data_ptr(), draft.data_ptr(), dt, parent.data_ptr(), tokens.data_ptr(),
                                       keep.data_ptr() if keep is not None else None, temperature.data_ptr(),
                                       u_accept.data_ptr(), u_resample.data_ptr(), B, N, V, nodes.data_ptr(),
                                       toks.data_ptr(), n.data_ptr(),
                                       log_norm.data_ptr() if log_norm is not None else None,
                                       status.data_ptr() if status is not None else None, s.cuda_stream))
    out = (nodes, toks, n)
    if return_log_norm:
        out += (log_norm,)
    if return_row_status:
        out += (status,)
    return out


def tree_prune(draft: torch.Tensor, parent: torch.Tensor, tokens: torch.Tensor, temperature: torch.Tensor,
               threshold: float, *, stream: torch.cuda.Stream | None = None):
    """Cumulative draft log-probability of every node and the keep mask at
    ``threshold``: (keep [B, N] int32, cum [B, N] float64), on the GPU."""
    lib = load_library()
    device = draft.device
    B, N, V = draft.shape
    dt = _dt_code(draft.dtype)
    _check(draft, "draft", None, (B, N, V), device)
    _check(parent, "parent", torch.int32, (B, N), device)
    _check(tokens, "tokens", torch.int32, (B, N), device)
    _check(temperature, "temperature", torch.float32, (B,), device)
    keep = torch.empty((B, N), dtype=torch.int32, device=device)
    cum = torch.empty((B, N), dtype=torch.float64, device=device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_tree_prune(draft.data_ptr(), dt, parent.data_ptr(), tokens.data_ptr(),
                                             temperature.data_ptr(), float(threshold), B, N, V, keep.data_ptr(),
                                             cum.data_ptr(), s.cuda_stream))
    return keep, cum


def _bf16_2d(t, name, shape, device):
    _check(t, name, torch.bfloat16, shape, device)


def lowrank_down(h: torch.Tensor, w_down: torch.Tensor, *, error: torch.Tensor | None = None,
                 stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """u = bf16(h W_down^T) on the tensor cores: h [M, d], W_down [r, d] bf16 -> [M, r]."""
    lib = load_library()
    device = h.device
    M, d = h.shape
    r = w_down.shape[0]
    _bf16_2d(h, "h", (M, d), device)
    _bf16_2d(w_down, "w_down", (r, d), device)
    u = torch.empty((M, r), dtype=torch.bfloat16, device=device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_lowrank_down(h.data_ptr(), w_down.data_ptr(), M, d, r, u.data_ptr(),
                                               error.data_ptr() if error is not None else None, s.cuda_stream))
    return u


def lowrank_up(u: torch.Tensor, w_up: torch.Tensor, temperature: torch.Tensor | None = None, *,
               with_lse: bool = True, error: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None):
    """z = bf16(u W_up^T) [M, V] and (with_lse) each row's log-normaliser at its temperature."""
    lib = load_library()
    device = u.device
    M, r = u.shape
    V = w_up.shape[0]
    _bf16_2d(u, "u", (M, r), device)
    _bf16_2d(w_up, "w_up", (V, r), device)
    if temperature is not None:
        _check(temperature, "temperature", torch.float32, (M,), device)
    z = torch.empty((M, V), dtype=torch.bfloat16, device=device)
    lse = torch.empty((M,), dtype=torch.float64, device=device) if with_lse else None
    ws = torch.empty(lib.spec_verify_lowrank_workspace_size(M, r, V), dtype=torch.uint8, device=device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_lowrank_up(u.data_ptr(), w_up.data_ptr(), M, r, V,
                                             temperature.data_ptr() if temperature is not None else None,
                                             z.data_ptr(), lse.data_ptr() if lse is not None else None,
                                             ws.data_ptr(), ws.numel(), error.data_ptr() if error is not None else None,
                                             s.cuda_stream))
    return (z, lse) if with_lse else z


def lowrank_head(h: torch.Tensor, w_down: torch.Tensor, w_up: torch.Tensor, temperature: torch.Tensor | None = None,
                 *, error: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                 stream: torch.cuda.Stream | None = None):
    """The low-rank draft head: (z [M, V] bf16 logits, lse [M] float64)."""
    lib = load_library()
    device = h.device
    M, d = h.shape
    r = w_down.shape[0]
    V = w_up.shape[0]
    _bf16_2d(h, "h", (M, d), device)
    _bf16_2d(w_down, "w_down", (r, d), device)
    _bf16_2d(w_up, "w_up", (V, r), device)
    if temperature is not None:
        _check(temperature, "temperature", torch.float32, (M,), device)
    z = torch.empty((M, V), dtype=torch.bfloat16, device=device)
    lse = torch.empty((M,), dtype=torch.float64, device=device)
    if workspace is None:
        workspace = torch.empty(lib.spec_verify_lowrank_workspace_size(M, r, V), dtype=torch.uint8, device=device)
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        _raise_if(lib.spec_verify_lowrank_head(h.data_ptr(), w_down.data_ptr(), w_up.data_ptr(), M, d, r, V,
                                               temperature.data_ptr() if temperature is not None else None,
                                               z.data_ptr(), lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                               error.data_ptr() if error is not None else None, s.cuda_stream))
    return z, lse


def lowrank_to_device(w, device="cuda"):
    """Copy a ``workloads.LowRankWorkload`` to torch tensors on ``device``."""
    def bf(a):
        return torch.from_numpy(a).view(torch.bfloat16).to(device)
    return dict(h=bf(w.h), w_down=bf(w.w_down), w_up=bf(w.w_up), temperature=torch.from_numpy(w.temperature).to(device))


def tree_to_device(w, device="cuda"):
    """Copy a ``workloads.TreeWorkload`` (numpy) to torch tensors on ``device``."""
    def logits(a):
        t = torch.from_numpy(a)
        if w.dtype == "bf16":
            t = t.view(torch.bfloat16)
        return t.to(device)
    return dict(target=logits(w.target), draft=logits(w.draft), parent=torch.from_numpy(w.parent).to(device),
                tokens=torch.from_numpy(w.tokens).to(device), temperature=torch.from_numpy(w.temperature).to(device),
                u_accept=torch.from_numpy(w.u_accept).to(device), u_resample=torch.from_numpy(w.u_resample).to(device))


def to_device(w, device="cuda"):
    """Copy a ``workloads.Workload`` (numpy) to torch tensors on ``device``."""
    def logits(a):
        t = torch.from_numpy(a)
        if w.dtype == "bf16":
            t = t.view(torch.bfloat16)
        return t.to(device)
    return dict(target=logits(w.target), draft=logits(w.draft),
                draft_tokens=torch.from_numpy(w.draft_tokens).to(device),
                temperature=torch.from_numpy(w.temperature).to(device),
                u_accept=torch.from_numpy(w.u_accept).to(device),
                u_resample=torch.from_numpy(w.u_resample).to(device))
