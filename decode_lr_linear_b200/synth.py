"""Seeded synthetic inputs for the low-rank decode path.

This module builds the tensors that both the CUDA library and the CPU oracle
consume: factor pairs, rank vectors, int8 weights with their scales, latent
K/V caches, queries and activations.  It performs only the *offline* steps
that turn random draws into stored model tensors (factorisation of a
synthetic spectrum, rotation folding, round-to-nearest weight quantisation,
rank allocation).  None of the runtime arithmetic of the decode path (the
GEMVs, dequantisation inside a product, SwiGLU, softmax, per-token requant)
lives here; that is written twice, once in ``oracle/`` and once in the CUDA
kernels, and the two share nothing but the arrays produced below.

Layout convention for stored factors (the library's ABI): both factors are
stored latent-major, one contiguous row per latent component j:
  * ``At``: [rank, d_in]  -- row j is column j of A (A is d_in x rank),
  * ``B``:  [rank, d_out] -- row j is row j of B (B is rank x d_out),
so that y = (x @ A) @ B = sum_j (x . At[j]) B[j].

Random draws: every large Gaussian array is filled in fixed-size chunks, each
from its own child of ``numpy.random.SeedSequence(seed, spawn_key=key)``, so
results do not depend on the number of threads used to fill them.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

_CHUNK = 1 << 22  # elements per independently seeded chunk


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


def normals(shape, seed: int, key: tuple, dtype=np.float32) -> np.ndarray:
    """Standard normal array of ``shape``, reproducible from (seed, key)."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=dtype)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    children = np.random.SeedSequence(seed, spawn_key=tuple(key)).spawn(nchunks)

    def fill(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        np.random.default_rng(children[i]).standard_normal(hi - lo, dtype=dtype, out=out[lo:hi])

    if nchunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


def rng_for(seed: int, key: tuple) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence(seed, spawn_key=tuple(key)))


def haar_orthogonal(n: int, rng: np.random.Generator, m: int | None = None) -> np.ndarray:
    """n x m (default n x n) matrix with orthonormal columns, Haar distributed.

    QR of a Gaussian matrix with the signs of R's diagonal moved into Q
    (Mezzadri, "How to generate random matrices from the classical compact
    groups", Notices AMS 2007), in float64.
    """
    m = n if m is None else m
    g = rng.standard_normal((n, m))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def harmonic(n: int) -> float:
    return float(sum(1.0 / i for i in range(1, n + 1)))


def to_bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.ascontiguousarray(a)).to(torch.bfloat16)


# --------------------------------------------------------------------------
# Single low-rank linear, fp32: d_in = d_out = 256, rank 32, one token.
# --------------------------------------------------------------------------
def make_single_linear(seed: int = 0, d: int = 256, rank: int = 32, exact_rank: bool = False) -> dict:
    """W = U diag(sigma) V^T with Haar U, V and sigma_i = i^-1/2.

    A = U_r diag(sigma_r)^1/2, B = diag(sigma_r)^1/2 V_r^T.  With
    ``exact_rank`` the spectrum beyond ``rank`` is zero, so W == A B exactly
    (up to fp64 rounding of the product).
    """
    rng = rng_for(seed, (1,))
    U = haar_orthogonal(d, rng)
    V = haar_orthogonal(d, rng)
    sigma = 1.0 / np.sqrt(np.arange(1, d + 1, dtype=np.float64))
    if exact_rank:
        sigma[rank:] = 0.0
    W = (U * sigma[None, :]) @ V.T  # d_in x d_out (math layout, y = x W)
    sr = np.sqrt(sigma[:rank])
    A = U[:, :rank] * sr[None, :]
    B = sr[:, None] * V[:, :rank].T
    x = rng.standard_normal((1, d))
    At32 = np.ascontiguousarray(A.T.astype(np.float32))
    B32 = np.ascontiguousarray(B.astype(np.float32))
    return {
        "U": U, "V": V, "sigma": sigma, "W": W, "A": A, "B": B,
        "At": torch.from_numpy(At32), "B32": torch.from_numpy(B32),
        "x": torch.from_numpy(x.astype(np.float32)),
        "d_in": d, "d_out": d, "rank": rank,
    }


# --------------------------------------------------------------------------
# Rank vectors
# --------------------------------------------------------------------------
def allocate_ranks(alpha: np.ndarray, cost: np.ndarray, budget: float, lo: np.ndarray, hi: np.ndarray,
                   quantum: int = 32) -> np.ndarray:
    """Non-uniform ranks from synthetic importances.

    r_p = round(alpha_p / S * R) with S = sum(alpha) and R chosen so that the
    parameter count sum_p r_p * cost_p meets ``budget`` (the proportional
    rule of FLRC, "Fisher-based layer-wise rank allocation"), clipped to
    [lo, hi] and rounded to multiples of ``quantum``; the rounding remainder
    is then moved one quantum at a time onto the entries with most slack
    until the budget is met to within one quantum of the cheapest entry.
    """
    alpha = np.asarray(alpha, np.float64)
    cost = np.asarray(cost, np.float64)
    lo = np.asarray(lo, np.float64)
    hi = np.asarray(hi, np.float64)
    S = alpha.sum()

    def ranks_for(R):
        r = np.clip(alpha / S * R, lo, hi)
        return np.clip(np.round(r / quantum) * quantum, np.ceil(lo / quantum) * quantum,
                       np.floor(hi / quantum) * quantum)

    # bisection on the total rank budget R
    a, b = 0.0, float(hi.sum()) * 4
    for _ in range(200):
        m = 0.5 * (a + b)
        if (ranks_for(m) * cost).sum() < budget:
            a = m
        else:
            b = m
    r = ranks_for(b)
    lo_q = np.ceil(lo / quantum) * quantum
    hi_q = np.floor(hi / quantum) * quantum
    # greedy fix-up towards the budget
    for _ in range(100000):
        err = budget - (r * cost).sum()
        if err >= 0:
            slack = hi_q - r
            cand = np.where(slack >= quantum)[0]
            if len(cand) == 0:
                break
            step_cost = quantum * cost[cand]
            ok = cand[step_cost <= err + 1e-9]
            if len(ok) == 0:
                break
            i = ok[np.argmax(slack[ok])]
            r[i] += quantum
        else:
            slack = r - lo_q
            cand = np.where(slack >= quantum)[0]
            if len(cand) == 0:
                break
            i = cand[np.argmax(slack[cand])]
            r[i] -= quantum
    return r.astype(np.int64)


ATTN_PROJ = ("q", "k", "v", "o")


def attention_ranks(seed: int = 0, layers: int = 32, hidden: int = 4096,
                    lo: int = 512, hi: int = 1536, keep: float = 0.6) -> np.ndarray:
    """[layers, 4] ranks for Q/K/V/O, in [lo, hi], multiples of 32.

    Synthetic importances alpha ~ LogNormal(0, 0.35); total factor parameters
    sum_p r_p (d_in + d_out) = keep * sum_p d_in d_out (40 % reduction for
    keep = 0.6), to within one rank quantum.
    """
    rng = rng_for(seed, (2, 0))
    n = layers * 4
    alpha = rng.lognormal(0.0, 0.35, size=n)
    cost = np.full(n, 2.0 * hidden)
    budget = keep * n * hidden * hidden
    r = allocate_ranks(alpha, cost, budget, np.full(n, lo), np.full(n, hi))
    return r.reshape(layers, 4)


def _lr_factors(d_in: int, d_out: int, rank: int, seed: int, key: tuple):
    """Gaussian-column factor pair with a decaying spectrum.

    A = G_A / sqrt(d_in) diag(sigma)^1/2, B = diag(sigma)^1/2 G_B / sqrt(d_out),
    sigma_i = c i^-1/2 with c = sqrt(d_out / H_rank), which gives
    Var(y_k) = 1 for x ~ N(0, I).  Returns (At [rank, d_in], B [rank, d_out]) float32.
    """
    sig = math.sqrt(d_out / harmonic(rank)) / np.sqrt(np.arange(1, rank + 1, dtype=np.float64))
    sq = np.sqrt(sig).astype(np.float32)
    At = normals((rank, d_in), seed, key + (0,))
    At *= (sq / np.float32(math.sqrt(d_in)))[:, None]
    B = normals((rank, d_out), seed, key + (1,))
    B *= (sq / np.float32(math.sqrt(d_out)))[:, None]
    return At, B


def make_attention_layer(layer: int, ranks: np.ndarray, seed: int = 0, hidden: int = 4096) -> dict:
    """bf16 factors of one layer's Q/K/V/O projections (LLaMA-7B shapes)."""
    out = {}
    for p, name in enumerate(ATTN_PROJ):
        At, B = _lr_factors(hidden, hidden, int(ranks[layer, p]), seed, (2, 1, layer, p))
        out[name] = {"At": to_bf16(At), "B": to_bf16(B), "rank": int(ranks[layer, p]),
                     "d_in": hidden, "d_out": hidden}
    return out


def make_activations(batch: int, dim: int, seed: int, key: tuple, outliers: int = 0,
                     outlier_scale: float = 20.0) -> torch.Tensor:
    """x ~ N(0, 1) [batch, dim] as bf16; ``outliers`` seeded channels scaled by 20 for every token."""
    x = normals((batch, dim), seed, key)
    if outliers:
        ch = rng_for(seed, key + (99,)).choice(dim, size=outliers, replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    return to_bf16(x)


# --------------------------------------------------------------------------
# Round-to-nearest int8 weights with per-output-channel scales.
# --------------------------------------------------------------------------
def rtn_int8_rows(Wt: np.ndarray, scale_dtype=np.float16):
    """Symmetric RTN with one scale per row (rows are the output channels).

    s = max|w| / 127 rounded to ``scale_dtype``; q = clamp(rint(w / s), -127, 127)
    against the rounded s (ties to even); s == 0 gives q == 0.
    """
    Wt = np.asarray(Wt, np.float64)
    amax = np.abs(Wt).max(axis=1)
    s = (amax / 127.0).astype(scale_dtype)
    s64 = s.astype(np.float64)
    safe = np.where(s64 > 0, s64, 1.0)
    q = np.clip(np.rint(Wt / safe[:, None]), -127, 127)
    q[s64 == 0] = 0
    return q.astype(np.int8), s


def rtn_int8_cols(W: np.ndarray, scale_dtype=np.float16):
    """Symmetric RTN with one scale per column (columns are the output channels)."""
    q, s = rtn_int8_rows(np.asarray(W).T, scale_dtype)
    return np.ascontiguousarray(q.T), s


def hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two)."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    assert h.shape[0] == n
    return h


def make_rotation(r: int, seed: int, block: int = 512) -> np.ndarray:
    """R = P blockdiag(H_block, ...)/sqrt(block) D: a seeded Hadamard-style orthogonal r x r."""
    assert r % block == 0
    rng = rng_for(seed, (3, 7))
    Hb = hadamard(block) / math.sqrt(block)
    Hfull = np.zeros((r, r))
    for i in range(r // block):
        Hfull[i * block:(i + 1) * block, i * block:(i + 1) * block] = Hb
    D = rng.choice([-1.0, 1.0], size=r)
    perm = rng.permutation(r)
    return (Hfull * D[None, :])[perm, :]


def make_hybrid_ffn(seed: int = 0, hidden: int = 4096, inter: int = 11008, n_lr: int = 8192,
                    rank: int = 1536, rotate: bool = True) -> dict:
    """Hybrid SwiGLU FFN weights (LLaMA-7B shape).

    The first ``n_lr`` hidden channels (a seeded permutation of the original
    channel order, folded offline into the stored weights) are low-rank:
    [W_gate[:, S] | W_up[:, S]] ~= A B with one shared latent of width
    ``rank``; the remaining inter - n_lr channels are dense.  The rotation R
    is folded as A' = A R, B' = R^T B, then every stored matrix is RTN int8
    with an fp16 scale per output channel.

    Stored tensors (int8; every scale belongs to one output channel):
      A_q  [rank, hidden]        s_A  [rank]       latent-major (row j = latent channel j)
      B_q  [rank, 2*n_lr]        s_B  [2*n_lr]     latent-major; columns interleaved gate0, up0, gate1, up1, ...
      D_q  [2*n_dense, hidden]   s_D  [2*n_dense]  output-major; rows interleaved gate0, up0, ...
      Wd_q [inter, hidden]       s_d  [hidden]     input-major; rows in [S; D] channel order
    """
    n_dense = inter - n_lr
    key = (3,)
    out = {"hidden": hidden, "inter": inter, "n_lr": n_lr, "n_dense": n_dense, "rank": rank}
    if n_lr > 0:
        At, B = _lr_factors(hidden, 2 * n_lr, rank, seed, key + (1,))
        At = At.astype(np.float64)
        B = B.astype(np.float64)
        if rotate:
            R = make_rotation(rank, seed)
            # A' = A R  ->  A'^T = R^T A^T ;  B' = R^T B
            At = R.T @ At
            B = R.T @ B
        qA, sA = rtn_int8_rows(At)
        qB, sB = rtn_int8_cols(B)
    else:
        qA = np.zeros((rank, hidden), np.int8); sA = np.zeros(rank, np.float16)
        qB = np.zeros((rank, 0), np.int8); sB = np.zeros(0, np.float16)
    Dt = normals((2 * n_dense, hidden), seed, key + (2,)) / np.float32(math.sqrt(hidden))
    qD, sD = rtn_int8_rows(Dt)
    Wd = normals((inter, hidden), seed, key + (3,)) / np.float32(math.sqrt(inter))
    qd, sd = rtn_int8_cols(Wd)
    for name, arr in (("A_q", qA), ("s_A", sA), ("B_q", qB), ("s_B", sB), ("D_q", qD), ("s_D", sD),
                      ("Wd_q", qd), ("s_d", sd)):
        out[name] = torch.from_numpy(np.ascontiguousarray(arr))
    return out


# --------------------------------------------------------------------------
# Per-head latent K/V caches.
# --------------------------------------------------------------------------
def make_latent_factors(heads: int, rank: int, head_dim: int, seed: int, key: tuple, peak: float = 1.0):
    """[heads, rank, head_dim] factors U diag(sigma) V^T, U rank x rank Haar,
    V head_dim x rank orthonormal, sigma_i = c i^-1/2, c = peak * sqrt(head_dim / H_rank)."""
    rng = rng_for(seed, key)
    c = peak * math.sqrt(head_dim / harmonic(rank))
    sig = c / np.sqrt(np.arange(1, rank + 1, dtype=np.float64))
    out = np.empty((heads, rank, head_dim))
    for h in range(heads):
        U = haar_orthogonal(rank, rng)
        V = haar_orthogonal(head_dim, rng, rank)
        out[h] = (U * sig[None, :]) @ V.T
    return out


def make_latent_kv(batch: int = 8, heads: int = 32, ctx: int = 4096, rank: int = 32, head_dim: int = 128,
                   seed: int = 0, seq_lens=None, peak: float = 1.0) -> dict:
    """bf16 latent caches C_K, C_V [batch, heads, ctx, rank] ~ N(0,1), factors B_K, B_V
    [heads, rank, head_dim] (bf16), query q [batch, heads, head_dim] ~ N(0,1) (bf16),
    seq_lens [batch] int32 (all ``ctx`` unless given)."""
    key = (4, ctx, batch, heads)
    CK = normals((batch, heads, ctx, rank), seed, key + (0,))
    CV = normals((batch, heads, ctx, rank), seed, key + (1,))
    q = normals((batch, heads, head_dim), seed, key + (2,))
    BK = make_latent_factors(heads, rank, head_dim, seed, key + (3,), peak)
    BV = make_latent_factors(heads, rank, head_dim, seed, key + (4,), 1.0)
    if seq_lens is None:
        seq_lens = np.full(batch, ctx, np.int32)
    return {"C_K": to_bf16(CK), "C_V": to_bf16(CV), "q": to_bf16(q),
            "B_K": to_bf16(BK), "B_V": to_bf16(BV),
            "seq_lens": torch.as_tensor(np.asarray(seq_lens, np.int32)),
            "batch": batch, "heads": heads, "ctx": ctx, "rank": rank, "head_dim": head_dim,
            "scale": 1.0 / math.sqrt(head_dim)}


def make_latent_kv_int8(batch: int = 8, heads: int = 32, ctx: int = 4096, rank: int = 32, head_dim: int = 128,
                        seed: int = 0, seq_lens=None, scale_dtype=np.float16) -> dict:
    """int8 latent caches with one positive scale per (batch, head, position): codes C_Kq, C_Vq
    [batch, heads, ctx, rank] drawn as rint(N(0,1) * 127 / 4) clipped to +-127, scales s_K, s_V
    [batch, heads, ctx] ~ 4/127 * U(0.5, 1.5) in ``scale_dtype``; B_K, B_V, q and seq_lens as
    make_latent_kv (the decode's inputs, as a cache writer would have left them)."""
    key = (6, ctx, batch, heads)
    out = make_latent_kv(batch=batch, heads=heads, ctx=1, rank=rank, head_dim=head_dim, seed=seed)
    for name, k in (("C_Kq", 0), ("C_Vq", 1)):
        g = normals((batch, heads, ctx, rank), seed, key + (k,))
        out[name] = torch.from_numpy(np.clip(np.rint(g * (127.0 / 4.0)), -127, 127).astype(np.int8))
    for name, k in (("s_K", 2), ("s_V", 3)):
        u = rng_for(seed, key + (k,)).uniform(0.5, 1.5, size=(batch, heads, ctx))
        out[name] = torch.from_numpy((u * 4.0 / 127.0).astype(scale_dtype))
    q = normals((batch, heads, head_dim), seed, key + (4,))
    out["q"] = to_bf16(q)
    if seq_lens is None:
        seq_lens = np.full(batch, ctx, np.int32)
    out["seq_lens"] = torch.as_tensor(np.asarray(seq_lens, np.int32))
    out["ctx"] = ctx
    del out["C_K"], out["C_V"]
    return out


def make_latent_producer(heads: int = 32, rank: int = 32, hidden: int = 4096, seed: int = 0) -> dict:
    """First factors of the per-head key/value projections, latent-major and stacked:
    A_KV [2 * heads * rank, hidden] bf16 ~ N(0, 1/hidden) (rows h*rank + j: A_Kh column j;
    rows (heads + h)*rank + j: A_Vh column j), so a latent of an N(0,1) token is O(1)."""
    A = normals((2 * heads * rank, hidden), seed, (7, heads, rank, hidden)) / math.sqrt(hidden)
    return {"A_KV": to_bf16(A), "heads": heads, "rank": rank, "hidden": hidden}


# --------------------------------------------------------------------------
# W8A8 prefill (LLaMA-13B shapes).
# --------------------------------------------------------------------------
PREFILL_PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def prefill_shapes(hidden: int = 5120, inter: int = 13824):
    return {"q": (hidden, hidden), "k": (hidden, hidden), "v": (hidden, hidden), "o": (hidden, hidden),
            "gate": (hidden, inter), "up": (hidden, inter), "down": (inter, hidden)}


def prefill_ranks(seed: int = 0, layers: int = 40, hidden: int = 5120, inter: int = 13824,
                  keep: float = 0.6) -> np.ndarray:
    """[layers, 7] ranks (multiples of 32) in [0.3, 0.9] x break-even with
    sum_p r_p (d_in + d_out) = keep * sum_p d_in d_out."""
    shp = prefill_shapes(hidden, inter)
    rng = rng_for(seed, (5, 0))
    n = layers * 7
    alpha = rng.lognormal(0.0, 0.35, size=n)
    d_in = np.array([shp[p][0] for p in PREFILL_PROJ] * layers, np.float64)
    d_out = np.array([shp[p][1] for p in PREFILL_PROJ] * layers, np.float64)
    be = d_in * d_out / (d_in + d_out)
    budget = keep * float((d_in * d_out).sum())
    r = allocate_ranks(alpha * be, d_in + d_out, budget, 0.3 * be, 0.9 * be)
    return r.reshape(layers, 7)


def make_prefill_projection(d_in: int, d_out: int, rank: int, seed: int, key: tuple) -> dict:
    """int8 factors with fp32 per-output-channel scales, latent-major:
    A_q [rank, d_in] s_A [rank], B_q [rank, d_out] s_B [d_out]."""
    At, B = _lr_factors(d_in, d_out, rank, seed, (5, 1) + tuple(key))
    qA, sA = rtn_int8_rows(At, np.float32)
    qB, sB = rtn_int8_cols(B, np.float32)
    return {"A_q": torch.from_numpy(qA), "s_A": torch.from_numpy(sA), "B_q": torch.from_numpy(qB),
            "s_B": torch.from_numpy(sB), "d_in": d_in, "d_out": d_out, "rank": rank}
