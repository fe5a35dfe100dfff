"""Torch-facing binding of the C ABI: same names as include/lr.h, argument marshalling only.

Each function turns torch tensors into device pointers and sizes, allocates
outputs and workspaces with torch when the caller passes none, and calls the
library on the current CUDA stream.  Every step of the computation runs in
the library's kernels; a missing library raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

from . import _lib as L

_DT = {torch.float32: L.LR_F32, torch.bfloat16: L.LR_BF16, torch.float16: L.LR_F16, torch.int8: L.LR_I8,
       torch.int32: L.LR_I32}


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


@dataclass
class Factor:
    """One factorised linear: A [rank, d_in] and B [rank, d_out], latent-major."""
    A: torch.Tensor
    B: torch.Tensor
    scale_A: Optional[torch.Tensor] = None
    scale_B: Optional[torch.Tensor] = None
    active_rank: int = 0

    @property
    def d_in(self) -> int:
        return self.A.shape[1]

    @property
    def d_out(self) -> int:
        return self.B.shape[1]

    @property
    def rank(self) -> int:
        return self.A.shape[0]

    def desc(self) -> L.FactorDesc:
        sd = _DT[self.scale_A.dtype] if self.scale_A is not None else L.LR_F32
        return L.FactorDesc(_ptr(self.A), _ptr(self.B), self.d_in, self.d_out, self.rank, self.active_rank,
                            _DT[self.A.dtype], sd, _ptr(self.scale_A), _ptr(self.scale_B))

    def out_dtype(self) -> torch.dtype:
        return torch.float32 if self.A.dtype == torch.float32 else torch.bfloat16


@dataclass
class FfnWeights:
    hidden: int
    inter: int
    n_lr: int
    rank: int
    A: torch.Tensor
    s_A: torch.Tensor
    B: torch.Tensor
    s_B: torch.Tensor
    D: torch.Tensor
    s_D: torch.Tensor
    W_down: torch.Tensor
    s_down: torch.Tensor

    def desc(self) -> L.FfnDesc:
        return L.FfnDesc(self.hidden, self.inter, self.n_lr, self.rank, _DT[self.s_down.dtype],
                         _ptr(self.A), _ptr(self.s_A), _ptr(self.B), _ptr(self.s_B),
                         _ptr(self.D) if self.D.numel() else None, _ptr(self.s_D) if self.s_D.numel() else None,
                         _ptr(self.W_down), _ptr(self.s_down))


@dataclass
class LatentKv:
    batch: int
    heads: int
    max_ctx: int
    B_K: torch.Tensor
    B_V: torch.Tensor
    scale: float
    mode: int = L.LR_KV_ABSORBED
    split_tokens: int = 0
    rope_base: float = 0.0
    rank: int = field(init=False)
    head_dim: int = field(init=False)

    def __post_init__(self):
        self.rank, self.head_dim = self.B_K.shape[1], self.B_K.shape[2]

    def desc(self, cache_scale_dtype: int = L.LR_F16) -> L.LatentKvDesc:
        return L.LatentKvDesc(self.batch, self.heads, self.head_dim, self.rank, self.max_ctx, self.scale,
                              _ptr(self.B_K), _ptr(self.B_V), self.mode, self.split_tokens, cache_scale_dtype,
                              self.rope_base)


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled workspace buffer (16-byte aligned, as torch allocations are)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def lr_linear_workspace_size(factor: Factor, batch: int, w8a8: bool = False) -> int:
    n = ctypes.c_size_t(0)
    d = factor.desc()
    L.check("lr_linear_workspace_size", L.load().lr_linear_workspace_size(ctypes.byref(d), batch, int(w8a8),
                                                                         ctypes.byref(n)))
    return n.value


def lr_linear(factor: Factor, x: torch.Tensor, y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
              x_scale: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    batch = x.shape[0]
    if y is None:
        y = torch.empty(batch, factor.d_out, dtype=torch.bfloat16 if x_scale is not None else factor.out_dtype(),
                        device=x.device)
    if ws is None:
        ws = workspace(lr_linear_workspace_size(factor, batch, x_scale is not None), x.device)
    d = factor.desc()
    L.check("lr_linear", L.load().lr_linear(ctypes.byref(d), _ptr(x), _ptr(x_scale), batch, _ptr(y), _ptr(ws),
                                            ws.numel() * ws.element_size(), _stream(stream)))
    return y


def _desc_array(factors: Sequence[Factor]):
    arr = (L.FactorDesc * len(factors))()
    for i, f in enumerate(factors):
        arr[i] = f.desc()
    return arr


def lr_linear_grouped_workspace_size(factors: Sequence[Factor], batch: int) -> int:
    n = ctypes.c_size_t(0)
    arr = _desc_array(factors)
    L.check("lr_linear_grouped_workspace_size",
            L.load().lr_linear_grouped_workspace_size(arr, len(factors), batch, ctypes.byref(n)))
    return n.value


def lr_linear_grouped(factors: Sequence[Factor], x: torch.Tensor, ys: Optional[Sequence[torch.Tensor]] = None,
                      ws: Optional[torch.Tensor] = None, stream=None) -> list:
    batch = x.shape[0]
    if ys is None:
        ys = [torch.empty(batch, f.d_out, dtype=f.out_dtype(), device=x.device) for f in factors]
    if ws is None:
        ws = workspace(lr_linear_grouped_workspace_size(factors, batch), x.device)
    arr = _desc_array(factors)
    yp = (ctypes.c_void_p * len(factors))(*[_ptr(y) for y in ys])
    L.check("lr_linear_grouped", L.load().lr_linear_grouped(arr, len(factors), _ptr(x), batch, yp, _ptr(ws),
                                                            ws.numel() * ws.element_size(), _stream(stream)))
    return list(ys)


@dataclass
class ChainStep:
    """One step of lr_linear_chain: projections sharing one input, which is the
    chain input (input_step = -1) or output `input_proj` of an earlier step."""
    factors: Sequence[Factor]
    input_step: int = -1
    input_proj: int = 0
    ys: Optional[Sequence[torch.Tensor]] = None


def _chain_array(steps: Sequence[ChainStep]):
    arr = (L.ChainStep * len(steps))()
    for i, st in enumerate(steps):
        arr[i].n = len(st.factors)
        arr[i].input_step = st.input_step
        arr[i].input_proj = st.input_proj
        for p, f in enumerate(st.factors):
            arr[i].proj[p] = f.desc()
            arr[i].y[p] = _ptr(st.ys[p]) if st.ys is not None else None
    return arr


def lr_linear_chain_workspace_size(steps: Sequence[ChainStep], batch: int) -> int:
    n = ctypes.c_size_t(0)
    arr = _chain_array([ChainStep(s.factors, s.input_step, s.input_proj,
                                  s.ys if s.ys is not None else [torch.empty(0)] * len(s.factors)) for s in steps])
    for i in range(len(steps)):  # placeholder outputs: only the shapes matter here
        for p in range(arr[i].n):
            arr[i].y[p] = 16
    L.check("lr_linear_chain_workspace_size", L.load().lr_linear_chain_workspace_size(arr, len(steps), batch,
                                                                                     ctypes.byref(n)))
    return n.value


def lr_linear_chain(steps: Sequence[ChainStep], x: torch.Tensor, ws: Optional[torch.Tensor] = None,
                    stream=None) -> list:
    """Runs the chain in one launch; returns every step's output list."""
    batch = x.shape[0]
    for st in steps:
        if st.ys is None:
            st.ys = [torch.empty(batch, f.d_out, dtype=f.out_dtype(), device=x.device) for f in st.factors]
    if ws is None:
        ws = workspace(lr_linear_chain_workspace_size(steps, batch), x.device)
    arr = _chain_array(steps)
    L.check("lr_linear_chain", L.load().lr_linear_chain(arr, len(steps), _ptr(x), batch, _ptr(ws),
                                                        ws.numel() * ws.element_size(), _stream(stream)))
    return [list(st.ys) for st in steps]


def lr_swiglu_ffn_workspace_size(ffn: FfnWeights, batch: int) -> int:
    n = ctypes.c_size_t(0)
    d = ffn.desc()
    L.check("lr_swiglu_ffn_workspace_size", L.load().lr_swiglu_ffn_workspace_size(ctypes.byref(d), batch,
                                                                                 ctypes.byref(n)))
    return n.value


def lr_swiglu_ffn(ffn: FfnWeights, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    batch = x.shape[0]
    if y is None:
        y = torch.empty(batch, ffn.hidden, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = workspace(lr_swiglu_ffn_workspace_size(ffn, batch), x.device)
    d = ffn.desc()
    L.check("lr_swiglu_ffn", L.load().lr_swiglu_ffn(ctypes.byref(d), _ptr(x), batch, _ptr(y), _ptr(ws),
                                                    ws.numel() * ws.element_size(), _stream(stream)))
    return y


def lr_latent_kv_workspace_size(kv: LatentKv) -> int:
    n = ctypes.c_size_t(0)
    d = kv.desc()
    L.check("lr_latent_kv_workspace_size", L.load().lr_latent_kv_workspace_size(ctypes.byref(d), ctypes.byref(n)))
    return n.value


def lr_latent_kv_decode(kv: LatentKv, q: torch.Tensor, C_K: torch.Tensor, C_V: torch.Tensor,
                        seq_lens: torch.Tensor, out: Optional[torch.Tensor] = None,
                        ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(kv.batch, kv.heads, kv.head_dim, dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = workspace(lr_latent_kv_workspace_size(kv), q.device)
    d = kv.desc()
    L.check("lr_latent_kv_decode",
            L.load().lr_latent_kv_decode(ctypes.byref(d), _ptr(q), _ptr(C_K), _ptr(C_V), _ptr(seq_lens), _ptr(out),
                                         _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return out


def lr_latent_kv_append_workspace_size(kv: LatentKv, hidden: int) -> int:
    n = ctypes.c_size_t(0)
    d = kv.desc()
    L.check("lr_latent_kv_append_workspace_size",
            L.load().lr_latent_kv_append_workspace_size(ctypes.byref(d), int(hidden), ctypes.byref(n)))
    return n.value


def lr_latent_kv_append(kv: LatentKv, A_KV: torch.Tensor, x: torch.Tensor, pos: torch.Tensor, C_K: torch.Tensor,
                        C_V: torch.Tensor, ws: Optional[torch.Tensor] = None, use_ws: bool = True,
                        stream=None) -> None:
    """Write the new token's per-head latents x A_Kh, x A_Vh into C_K, C_V at position pos[b].

    With a workspace (allocated here when ``ws`` is None and ``use_ws``) the product runs on the tensor
    cores; ``use_ws=False`` keeps the CUDA-core GEMV."""
    hidden = A_KV.shape[1]
    if ws is None and use_ws:
        n = lr_latent_kv_append_workspace_size(kv, hidden)
        ws = workspace(n, x.device) if n else None
    d = kv.desc()
    L.check("lr_latent_kv_append",
            L.load().lr_latent_kv_append(ctypes.byref(d), _ptr(A_KV), hidden, _ptr(x), _ptr(pos), _ptr(C_K),
                                         _ptr(C_V), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                         _stream(stream)))


def lr_quantize_per_token(x: torch.Tensor, x_q: Optional[torch.Tensor] = None, s: Optional[torch.Tensor] = None,
                          stream=None):
    rows, cols = x.shape
    if x_q is None:
        x_q = torch.empty(rows, cols, dtype=torch.int8, device=x.device)
    if s is None:
        s = torch.empty(rows, dtype=torch.float32, device=x.device)
    L.check("lr_quantize_per_token", L.load().lr_quantize_per_token(_ptr(x), rows, cols, _ptr(x_q), _ptr(s),
                                                                    _stream(stream)))
    return x_q, s


def lr_gemm_s8s32(A: torch.Tensor, B: torch.Tensor, b_layout: int, C: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """C = A B (int8 x int8 -> int32).  b_layout 0: B is [N, K]; 1: B is [K, N]."""
    M, K = A.shape
    N = B.shape[0] if b_layout == 0 else B.shape[1]
    if C is None:
        C = torch.empty(M, N, dtype=torch.int32, device=A.device)
    L.check("lr_gemm_s8s32", L.load().lr_gemm_s8s32(_ptr(A), _ptr(B), b_layout, M, N, K, _ptr(C), _stream(stream)))
    return C


def lr_workspace_init(ws: torch.Tensor, stream=None) -> None:
    L.check("lr_workspace_init", L.load().lr_workspace_init(_ptr(ws), ws.numel() * ws.element_size(),
                                                            _stream(stream)))


def lr_check_device_error(stream=None) -> int:
    err = ctypes.c_int(0)
    st = L.load().lr_check_device_error(_stream(stream), ctypes.byref(err))
    if st not in (L.LR_OK, L.LR_ERR_DEVICE_TIMEOUT):
        raise L.LrError("lr_check_device_error", st)
    return err.value


def lr_set_wait_timeout_us(us: int) -> None:
    """Bound of a persistent kernel's waits on its other CTAs, in microseconds (0: default, 1 s)."""
    L.check("lr_set_wait_timeout_us", L.load().lr_set_wait_timeout_us(int(us)))


def lr_set_tensor_core_min_batch(linear: int = 0, ffn: int = 0) -> None:
    """Smallest batch that takes the tensor-core path (0: the default, 9)."""
    L.check("lr_set_tensor_core_min_batch", L.load().lr_set_tensor_core_min_batch(int(linear), int(ffn)))


def _rank_vec(values):
    arr = (ctypes.c_int * len(values))(*[int(v) for v in values])
    return L.RankVec(len(values), arr), arr


def lr_rank_allocate(alpha: Sequence[float], r_budget: float, caps: Sequence[int]) -> list:
    """FLRC ranks r_p = clamp(round(alpha_p / S * r_budget), 1, caps_p), computed by the library (host)."""
    n = len(alpha)
    a = (ctypes.c_double * n)(*[float(v) for v in alpha])
    cap, _keep = _rank_vec(caps)
    out = (ctypes.c_int * n)()
    L.check("lr_rank_allocate", L.load().lr_rank_allocate(a, n, float(r_budget), ctypes.byref(cap), out))
    return list(out)


def lr_linear_chain_ranked(steps: Sequence[ChainStep], x: torch.Tensor, active: Sequence[int],
                           ws: Optional[torch.Tensor] = None, stream=None) -> list:
    """lr_linear_chain with per-projection active ranks (chain order, 0 = every component)."""
    batch = x.shape[0]
    for st in steps:
        if st.ys is None:
            st.ys = [torch.empty(batch, f.d_out, dtype=f.out_dtype(), device=x.device) for f in st.factors]
    if ws is None:
        ws = workspace(lr_linear_chain_workspace_size(steps, batch), x.device)
    arr = _chain_array(steps)
    rv, _keep = _rank_vec(active)
    L.check("lr_linear_chain_ranked", L.load().lr_linear_chain_ranked(arr, len(steps), ctypes.byref(rv), _ptr(x), batch,
                                                                      _ptr(ws), ws.numel() * ws.element_size(),
                                                                      _stream(stream)))
    return [list(st.ys) for st in steps]


def lr_dense_linear(W: torch.Tensor, x: torch.Tensor, scale: Optional[torch.Tensor] = None,
                    y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense baseline y = x W_store^T for an output-major weight W_store [d_out, d_in] (bf16, or int8 + scale)."""
    d_out, d_in = W.shape
    batch = x.shape[0]
    if y is None:
        y = torch.empty(batch, d_out, dtype=torch.bfloat16, device=x.device)
    sd = _DT[scale.dtype] if scale is not None else L.LR_F32
    L.check("lr_dense_linear", L.load().lr_dense_linear(_ptr(W), _DT[W.dtype], _ptr(scale), sd, d_in, d_out, _ptr(x),
                                                        batch, _ptr(y), _stream(stream)))
    return y


def lr_flash_decode(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                    out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, split_tokens: int = 0,
                    stream=None) -> torch.Tensor:
    """Flash decoding over full K/V [batch, heads, max_ctx, 128] (the uncompressed baseline)."""
    batch, heads, max_ctx, hd = K.shape
    d = L.FlashDesc(batch, heads, hd, max_ctx, float(scale), split_tokens)
    if out is None:
        out = torch.empty(batch, heads, hd, dtype=torch.bfloat16, device=q.device)
    if ws is None:
        n = ctypes.c_size_t(0)
        L.check("lr_flash_decode_workspace_size", L.load().lr_flash_decode_workspace_size(ctypes.byref(d),
                                                                                          ctypes.byref(n)))
        ws = workspace(n.value, q.device)
    L.check("lr_flash_decode", L.load().lr_flash_decode(ctypes.byref(d), _ptr(q), _ptr(K), _ptr(V), _ptr(seq_lens),
                                                        _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                                        _stream(stream)))
    return out


def lr_latent_kv_decode_q8(kv: LatentKv, q: torch.Tensor, C_K: torch.Tensor, s_K: torch.Tensor, C_V: torch.Tensor,
                           s_V: torch.Tensor, seq_lens: torch.Tensor, out: Optional[torch.Tensor] = None,
                           ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Latent-KV decode over int8 caches with one scale per (batch, head, position)."""
    if out is None:
        out = torch.empty(kv.batch, kv.heads, kv.head_dim, dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = workspace(lr_latent_kv_workspace_size(kv), q.device)
    d = kv.desc(_DT[s_K.dtype])
    L.check("lr_latent_kv_decode_q8",
            L.load().lr_latent_kv_decode_q8(ctypes.byref(d), _ptr(q), _ptr(C_K), _ptr(s_K), _ptr(C_V), _ptr(s_V),
                                            _ptr(seq_lens), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)))
    return out
