"""The C-ABI library loads, exports what include/lr.h declares, and validates
arguments on the host (CPU only: no call here reaches a kernel launch)."""
import ctypes

import pytest

from decode_lr_linear_b200 import _lib as L

FAKE = 0x10000          # a 16-byte aligned non-null address (never dereferenced on the host)
MIS = 0x10001           # a misaligned address


@pytest.fixture(scope="module")
def lib():
    return L.load()


def test_every_declared_symbol_is_exported(lib):
    names = L.header_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(7):
        assert lib.lr_status_string(s)
    assert lib.lr_version() >= 100


def _desc(**kw):
    d = dict(A=FAKE, B=FAKE, d_in=4096, d_out=4096, rank=1024, active_rank=0, w_dtype=L.LR_BF16,
             scale_dtype=L.LR_F32, scale_A=None, scale_B=None)
    d.update(kw)
    return L.FactorDesc(**d)


def _ws(lib, d, batch, w8a8=0):
    n = ctypes.c_size_t(0)
    st = lib.lr_linear_workspace_size(ctypes.byref(d), batch, w8a8, ctypes.byref(n))
    return st, n.value


def test_linear_workspace_sizes(lib):
    # completion counters (256 bytes) + min(batch, 8) x d_out fp32 accumulators (8-rounded)
    st, n = _ws(lib, _desc(), 1)
    assert st == L.LR_OK and n == 256 + 4096 * 4
    st, n3 = _ws(lib, _desc(), 3)
    assert st == L.LR_OK and n3 == 256 + 3 * 4096 * 4
    # bf16 from batch 4 (tensor cores): two latent sets [cols, rank] and two y sets [cols, d_out],
    # cols = 8-rounded min(batch, 32); the larger of the two paths' needs
    st, n16 = _ws(lib, _desc(), 16)
    assert st == L.LR_OK and n16 == 256 + (2 * 1024 + 2 * 4096) * 16 * 4
    st, n40 = _ws(lib, _desc(), 40)
    assert st == L.LR_OK and n40 == 256 + (2 * 1024 + 2 * 4096) * 32 * 4
    st, n16f = _ws(lib, _desc(w_dtype=L.LR_F32), 16)
    assert st == L.LR_OK and n16f == 256 + 8 * 4096 * 4
    st, n3s = _ws(lib, _desc(d_out=8), 3)
    assert st == L.LR_OK and n3s == 256 + 24 * 4
    st, _ = _ws(lib, _desc(w_dtype=L.LR_I8), 1)
    assert st == L.LR_ERR_INVALID_ARG  # int8 needs scales
    # W8A8: int32 sums [batch, rp] + int8 latent [bp, rp] + f32 scales [bp] (rp, bp: 128-rounded; parts 256-rounded)
    st, n = _ws(lib, _desc(w_dtype=L.LR_I8, scale_A=FAKE, scale_B=FAKE), 2048, 1)
    assert st == L.LR_OK and n == 2048 * 1024 * 4 + 2048 * 1024 + 2048 * 4
    st, n = _ws(lib, _desc(w_dtype=L.LR_I8, scale_A=FAKE, scale_B=FAKE, active_rank=200), 130, 1)
    assert st == L.LR_OK and n == 130 * 256 * 4 + 256 * 256 + 1024


def test_linear_validation(lib):
    call = lambda d, x=FAKE, xs=None, b=1, y=FAKE, ws=FAKE, wsb=1 << 20: lib.lr_linear(  # noqa: E731
        ctypes.byref(d) if d is not None else None, x, xs, b, y, ws, wsb, None)
    assert call(None) == L.LR_ERR_INVALID_ARG
    assert call(_desc(A=None)) == L.LR_ERR_INVALID_ARG
    assert call(_desc(rank=0)) == L.LR_ERR_INVALID_ARG
    assert call(_desc(active_rank=2000)) == L.LR_ERR_INVALID_ARG
    assert call(_desc(d_in=4100)) == L.LR_ERR_UNSUPPORTED
    assert call(_desc(w_dtype=L.LR_F16)) == L.LR_ERR_UNSUPPORTED
    i8 = dict(w_dtype=L.LR_I8, scale_A=FAKE, scale_B=FAKE)
    assert call(_desc(d_in=4104, **i8)) == L.LR_ERR_UNSUPPORTED   # int8 rows must be 16-byte multiples
    assert call(_desc(d_in=16392)) == L.LR_ERR_UNSUPPORTED        # bf16 row above 32 KiB
    assert call(_desc(A=MIS)) == L.LR_ERR_MISALIGNED
    assert call(_desc(), x=MIS) == L.LR_ERR_MISALIGNED
    assert call(_desc(), b=0) == L.LR_ERR_INVALID_ARG
    assert call(_desc(), wsb=16) == L.LR_ERR_WORKSPACE
    assert call(_desc(), ws=None) == L.LR_ERR_WORKSPACE
    assert call(_desc(), xs=FAKE) == L.LR_ERR_UNSUPPORTED  # W8A8 needs int8 weights
    d8 = _desc(w_dtype=L.LR_I8, scale_A=FAKE, scale_B=FAKE, scale_dtype=L.LR_F16)
    assert call(d8, xs=FAKE) == L.LR_ERR_UNSUPPORTED  # W8A8 needs fp32 scales


def test_grouped_validation(lib):
    arr = (L.FactorDesc * 3)(_desc(), _desc(d_in=2048), _desc())
    ys = (ctypes.c_void_p * 3)(FAKE, FAKE, FAKE)
    assert lib.lr_linear_grouped(arr, 3, FAKE, 1, ys, FAKE, 1 << 20, None) == L.LR_ERR_INVALID_ARG
    arr = (L.FactorDesc * 5)(*[_desc()] * 5)
    assert lib.lr_linear_grouped(arr, 5, FAKE, 1, ys, FAKE, 1 << 20, None) == L.LR_ERR_INVALID_ARG
    arr = (L.FactorDesc * 3)(_desc(), _desc(d_out=1024), _desc(rank=512))
    n = ctypes.c_size_t(0)
    assert lib.lr_linear_grouped_workspace_size(arr, 3, 1, ctypes.byref(n)) == L.LR_OK
    assert n.value == 256 + (4096 + 1024 + 4096) * 4


def _ffn(**kw):
    d = dict(hidden=4096, inter=11008, n_lr=8192, rank=1536, scale_dtype=L.LR_F16, A=FAKE, s_A=FAKE, B=FAKE,
             s_B=FAKE, D=FAKE, s_D=FAKE, W_down=FAKE, s_down=FAKE)
    d.update(kw)
    return L.FfnDesc(**d)


def test_ffn_validation_and_workspace(lib):
    n = ctypes.c_size_t(0)
    d = _ffn()
    assert lib.lr_swiglu_ffn_workspace_size(ctypes.byref(d), 1, ctypes.byref(n)) == L.LR_OK
    # tensor-core path (every batch by default): 256 bytes, then per token (8 columns at batch 1)
    # z [rank], gate/up [2 inter], h [inter], y [hidden] fp32
    assert n.value == 256 + (1536 + 2 * 11008 + 11008 + 4096) * 8 * 4
    # the CUDA-core path's need: gate/up of the low-rank channels, h of the dense ones, y
    try:
        assert lib.lr_set_tensor_core_min_batch(64, 64) == L.LR_OK
        assert lib.lr_swiglu_ffn_workspace_size(ctypes.byref(d), 1, ctypes.byref(n)) == L.LR_OK
        assert n.value == 256 + 16384 * 4 + 2816 * 4 + 4096 * 4
    finally:
        lib.lr_set_tensor_core_min_batch(0, 0)
    bad = _ffn(n_lr=12000)
    assert lib.lr_swiglu_ffn(ctypes.byref(bad), FAKE, 1, FAKE, FAKE, 1 << 20, None) == L.LR_ERR_INVALID_ARG
    bad = _ffn(n_lr=8196)
    assert lib.lr_swiglu_ffn(ctypes.byref(bad), FAKE, 1, FAKE, FAKE, 1 << 20, None) == L.LR_ERR_UNSUPPORTED
    bad = _ffn(hidden=4100)
    assert lib.lr_swiglu_ffn(ctypes.byref(bad), FAKE, 1, FAKE, FAKE, 1 << 20, None) == L.LR_ERR_UNSUPPORTED
    bad = _ffn(D=MIS)
    assert lib.lr_swiglu_ffn(ctypes.byref(bad), FAKE, 1, FAKE, FAKE, 1 << 20, None) == L.LR_ERR_MISALIGNED
    assert lib.lr_swiglu_ffn(ctypes.byref(d), FAKE, 1, FAKE, FAKE, 64, None) == L.LR_ERR_WORKSPACE
    dense_only = _ffn(n_lr=0, A=None, s_A=None, B=None, s_B=None)
    assert lib.lr_swiglu_ffn_workspace_size(ctypes.byref(dense_only), 1, ctypes.byref(n)) == L.LR_OK


def _kv(**kw):
    d = dict(batch=8, heads=32, head_dim=128, rank=32, max_ctx=4096, scale=128 ** -0.5, B_K=FAKE, B_V=FAKE,
             mode=L.LR_KV_ABSORBED, split_tokens=0, cache_scale_dtype=L.LR_F16, rope_base=0.0)
    d.update(kw)
    return L.LatentKvDesc(**d)


def test_latent_kv_validation_and_workspace(lib):
    n = ctypes.c_size_t(0)
    d = _kv()
    assert lib.lr_latent_kv_workspace_size(ctypes.byref(d), ctypes.byref(n)) == L.LR_OK
    assert n.value == 8 * 32 * (4096 // 256) * 34 * 4 + 8 * 32 * 32 * 4   # partials + the projected queries
    for bad, code in ((_kv(rank=16), L.LR_ERR_UNSUPPORTED), (_kv(head_dim=64), L.LR_ERR_UNSUPPORTED),
                      (_kv(split_tokens=100), L.LR_ERR_INVALID_ARG), (_kv(batch=0), L.LR_ERR_INVALID_ARG),
                      (_kv(B_K=MIS), L.LR_ERR_MISALIGNED)):
        assert lib.lr_latent_kv_decode(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                       None) == code
    assert lib.lr_latent_kv_decode(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                                   None) == L.LR_ERR_WORKSPACE


def test_quantize_validation(lib):
    assert lib.lr_quantize_per_token(FAKE, 4, 100, FAKE, FAKE, None) == L.LR_ERR_UNSUPPORTED
    assert lib.lr_quantize_per_token(None, 4, 128, FAKE, FAKE, None) == L.LR_ERR_INVALID_ARG
    assert lib.lr_quantize_per_token(MIS, 4, 128, FAKE, FAKE, None) == L.LR_ERR_MISALIGNED


def _step(n=1, input_step=-1, input_proj=0, **kw):
    st = L.ChainStep()
    st.n, st.input_step, st.input_proj = n, input_step, input_proj
    for p in range(n):
        st.proj[p] = _desc(**kw)
        st.y[p] = FAKE
    return st


def test_chain_validation_and_workspace(lib):
    arr = (L.ChainStep * 3)(_step(3), _step(1, 0, 2), _step(3, 1, 0))
    n = ctypes.c_size_t(0)
    assert lib.lr_linear_chain_workspace_size(arr, 3, 1, ctypes.byref(n)) == L.LR_OK
    assert n.value == 256 + (3 + 1 + 3) * 4096 * 4     # counters + every step's own accumulators
    bad = (L.ChainStep * 2)(_step(1), _step(1, 1, 0))            # input from itself
    assert lib.lr_linear_chain(bad, 2, FAKE, 1, FAKE, 1 << 24, None) == L.LR_ERR_INVALID_ARG
    bad = (L.ChainStep * 2)(_step(1), _step(1, 0, 3))            # no such output
    assert lib.lr_linear_chain(bad, 2, FAKE, 1, FAKE, 1 << 24, None) == L.LR_ERR_INVALID_ARG
    bad = (L.ChainStep * 2)(_step(1), _step(1, 0, 0, d_in=2048))  # width mismatch
    assert lib.lr_linear_chain(bad, 2, FAKE, 1, FAKE, 1 << 24, None) == L.LR_ERR_INVALID_ARG
    assert lib.lr_linear_chain(arr, 3, FAKE, 1, FAKE, 64, None) == L.LR_ERR_WORKSPACE
    assert lib.lr_linear_chain(arr, 0, FAKE, 1, FAKE, 1 << 24, None) == L.LR_ERR_INVALID_ARG


def test_noalloc_validation_order(lib):
    # a row wider than 32 KiB is refused as unsupported, as lr_linear refuses it
    d = _desc(d_out=20000)
    assert lib.lr_linear_noalloc(ctypes.byref(d), FAKE, 1, FAKE, None) == L.LR_ERR_UNSUPPORTED
    # a valid shape whose scratch exceeds the fixed array: int8, d_out 32768, batch 8
    d = _desc(w_dtype=L.LR_I8, scale_A=FAKE, scale_B=FAKE, d_in=64, d_out=32768, rank=32)
    assert lib.lr_linear_noalloc(ctypes.byref(d), FAKE, 8, FAKE, None) == L.LR_ERR_WORKSPACE
    st, n = _ws(lib, d, 8)
    assert st == L.LR_OK and n > L.LR_NOALLOC_SCRATCH_BYTES


def test_wait_timeout_setter(lib):
    assert lib.lr_set_wait_timeout_us(500) == L.LR_OK
    assert lib.lr_set_wait_timeout_us(0) == L.LR_OK


def test_rank_allocate_matches_oracle_exactly(lib):
    # the library's FLRC rule on the host against the oracle, on random importances,
    # budgets and caps (integer results: bit-exact)
    import numpy as np

    import decode_lr_linear_b200 as lr
    from oracle import ranks
    rng = np.random.default_rng(5)
    for trial in range(200):
        n = int(rng.integers(1, 130))
        alpha = rng.lognormal(0.0, 0.6, n)
        caps = rng.integers(1, 2000, n)
        budget = float(rng.uniform(0, 3000 * n)) if trial % 7 else float(n) * 0.5
        assert lr.lr_rank_allocate(alpha, budget, caps) == ranks.flrc_ranks(alpha, budget, caps).tolist()


def test_rank_allocate_and_ranked_chain_validation(lib):
    a = (ctypes.c_double * 2)(1.0, -1.0)
    caps = (ctypes.c_int * 2)(10, 10)
    cap = L.RankVec(2, caps)
    out = (ctypes.c_int * 2)()
    assert lib.lr_rank_allocate(a, 2, 10.0, ctypes.byref(cap), out) == L.LR_ERR_INVALID_ARG   # alpha <= 0
    a = (ctypes.c_double * 2)(1.0, 1.0)
    assert lib.lr_rank_allocate(a, 2, -1.0, ctypes.byref(cap), out) == L.LR_ERR_INVALID_ARG   # negative budget
    bad_cap = L.RankVec(3, caps)
    assert lib.lr_rank_allocate(a, 2, 10.0, ctypes.byref(bad_cap), out) == L.LR_ERR_INVALID_ARG
    arr = (L.ChainStep * 2)(_step(3), _step(1, 0, 2))
    r = (ctypes.c_int * 3)(100, 200, 300)
    short = L.RankVec(3, r)                       # the chain has 4 projections
    assert lib.lr_linear_chain_ranked(arr, 2, ctypes.byref(short), FAKE, 1, FAKE, 1 << 24, None) == \
        L.LR_ERR_INVALID_ARG
    r4 = (ctypes.c_int * 4)(100, 200, 2000, 5)    # 2000 > stored rank 1024
    over = L.RankVec(4, r4)
    assert lib.lr_linear_chain_ranked(arr, 2, ctypes.byref(over), FAKE, 1, FAKE, 1 << 24, None) == \
        L.LR_ERR_INVALID_ARG


def test_dense_and_flash_validation(lib):
    assert lib.lr_dense_linear(FAKE, L.LR_F32, None, L.LR_F32, 4096, 4096, FAKE, 1, FAKE, None) == L.LR_ERR_UNSUPPORTED
    assert lib.lr_dense_linear(FAKE, L.LR_I8, None, L.LR_F32, 4096, 4096, FAKE, 1, FAKE, None) == L.LR_ERR_INVALID_ARG
    assert lib.lr_dense_linear(FAKE, L.LR_BF16, None, L.LR_F32, 4100, 4096, FAKE, 1, FAKE, None) == L.LR_ERR_UNSUPPORTED
    assert lib.lr_dense_linear(FAKE, L.LR_BF16, None, L.LR_F32, 32768, 8, FAKE, 1, FAKE, None) == L.LR_ERR_UNSUPPORTED
    assert lib.lr_dense_linear(MIS, L.LR_BF16, None, L.LR_F32, 4096, 8, FAKE, 1, FAKE, None) == L.LR_ERR_MISALIGNED
    d = L.FlashDesc(8, 32, 128, 4096, 0.088, 0)
    n = ctypes.c_size_t(0)
    assert lib.lr_flash_decode_workspace_size(ctypes.byref(d), ctypes.byref(n)) == L.LR_OK
    assert n.value == 8 * 32 * (4096 // 128) * 130 * 4
    for bad, code in ((L.FlashDesc(8, 32, 64, 4096, 0.1, 0), L.LR_ERR_UNSUPPORTED),
                      (L.FlashDesc(8, 32, 128, 4096, 0.1, 100), L.LR_ERR_INVALID_ARG),
                      (L.FlashDesc(8, 32, 128, 4096, 0.1, 512), L.LR_ERR_INVALID_ARG)):
        assert lib.lr_flash_decode(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == code
    assert lib.lr_flash_decode(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == L.LR_ERR_WORKSPACE


def test_latent_kv_q8_validation(lib):
    d = _kv()
    assert lib.lr_latent_kv_decode_q8(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                      None) == L.LR_ERR_INVALID_ARG
    bad = _kv(cache_scale_dtype=L.LR_BF16)
    assert lib.lr_latent_kv_decode_q8(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                      None) == L.LR_ERR_UNSUPPORTED
    assert lib.lr_latent_kv_decode_q8(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                                      None) == L.LR_ERR_WORKSPACE


def test_latent_kv_reconstruct_mode_validation(lib):
    # the on-chip reconstruction mode takes a rotary base; the absorbed form refuses one
    n = ctypes.c_size_t(0)
    rec = _kv(mode=L.LR_KV_RECONSTRUCT, rope_base=10000.0)
    assert lib.lr_latent_kv_workspace_size(ctypes.byref(rec), ctypes.byref(n)) == L.LR_OK
    assert n.value == 8 * 32 * (4096 // 256) * 34 * 4 + 8 * 32 * 32 * 4
    for bad, code in ((_kv(rope_base=10000.0), L.LR_ERR_UNSUPPORTED),
                      (_kv(mode=L.LR_KV_RECONSTRUCT, rope_base=-1.0), L.LR_ERR_INVALID_ARG),
                      (_kv(mode=L.LR_KV_RECONSTRUCT, rope_base=float("nan")), L.LR_ERR_INVALID_ARG),
                      (_kv(mode=L.LR_KV_RECONSTRUCT, split_tokens=512), L.LR_ERR_UNSUPPORTED),
                      (_kv(mode=L.LR_KV_RECONSTRUCT, batch=4096, heads=1024, max_ctx=1024), L.LR_ERR_UNSUPPORTED),
                      (_kv(mode=7), L.LR_ERR_UNSUPPORTED)):
        assert lib.lr_latent_kv_decode(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                       None) == code
    # int8 caches have no reconstruct mode
    assert lib.lr_latent_kv_decode_q8(ctypes.byref(rec), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                      None) == L.LR_ERR_UNSUPPORTED
    assert lib.lr_latent_kv_decode(ctypes.byref(rec), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                                   None) == L.LR_ERR_WORKSPACE


def test_latent_kv_append_validation(lib):
    d = _kv()
    app = lambda dd, a=FAKE, hid=4096, pos=FAKE, ws=None, wsb=0: lib.lr_latent_kv_append(  # noqa: E731
        ctypes.byref(dd), a, hid, FAKE, pos, FAKE, FAKE, ws, wsb, None)
    assert app(d, a=None) == L.LR_ERR_INVALID_ARG
    assert app(d, hid=0) == L.LR_ERR_INVALID_ARG
    assert app(d, hid=4100) == L.LR_ERR_UNSUPPORTED
    assert app(d, hid=32768) == L.LR_ERR_UNSUPPORTED
    assert app(d, pos=MIS) == L.LR_ERR_MISALIGNED
    assert app(_kv(batch=0)) == L.LR_ERR_INVALID_ARG
    # the tensor-core path's workspace: counters + a token-major fp32 row of 2 * heads * rank per token
    n = ctypes.c_size_t(0)
    assert lib.lr_latent_kv_append_workspace_size(ctypes.byref(d), 4096, ctypes.byref(n)) == L.LR_OK
    assert n.value == 256 + 2 * 32 * 32 * 8 * 4
    assert app(d, ws=FAKE, wsb=64) == L.LR_ERR_WORKSPACE
    assert app(d, ws=MIS, wsb=1 << 20) == L.LR_ERR_MISALIGNED
