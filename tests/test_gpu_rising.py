"""GPU parity when scores rise along the sequence (pa_testlib.rising_scores:
keys scaled by 1 + t / 256 at token t, query rows scaled by 0.05 .. 1.6), so
that a row's running max is passed by more than the kernels' lazy-rescale
gap in the middle of a sequence, for some rows of a tile and not others:
the reference moves and the partial output is rescaled mid-stream, in every
kernel family (tensor-core decode at blocks of 8, 16 and 32, the CUDA-core
kernel, multi-query token-major tiles, shared-prefix group units) and
across split units.  Against the float64 oracle, element by element:
max-abs 2e-3 where |oracle| < 0.5, max-rel 1e-2 where |oracle| >= 0.1."""

import numpy as np
import pytest

from pa_testlib import assert_attention_close, gpu_step, oracle_step, rising_scores, to_device, torch_f64
from workloads import fill_values_numpy, random_layout

pytestmark = pytest.mark.gpu

LENS = [1, 17, 300, 1000, 2500, 4100]

DECODE = [
    (4, 128, 16, "bf16", 0),   # tensor cores, Llama-3-8B grouping
    (1, 128, 16, "fp16", 0),   # tensor cores, MHA
    (8, 128, 8, "bf16", 37),   # 8-token blocks, split units
    (2, 128, 32, "fp16", 5),   # 32-token blocks, split units
    (4, 64, 16, "bf16", 0),    # CUDA cores (head_dim 64)
    (4, 64, 16, "fp16", 7),
]


@pytest.mark.parametrize("G,D,B,dtype,num_ctas", DECODE,
                         ids=[f"G{g}-D{d}-B{b}-{t}-ctas{n}" for g, d, b, t, n in DECODE])
def test_decode_rising_scores(cuda_device, G, D, B, dtype, num_ctas):
    seed = 8300 + 10 * G + B + D
    L = random_layout(seed, LENS, dtype=dtype, block_size=B, num_q_heads=2 * G, num_kv_heads=2, head_dim=D,
                      write_new_token=True)
    V0 = fill_values_numpy(L)
    V, q = rising_scores(L, V0, V0.q, seed)
    V.q = q
    out, st = gpu_step(to_device(L, V, cuda_device), L, num_ctas=num_ctas)
    assert int(st.item()) == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out), ref, f"rising decode G={G} D={D} B={B} {dtype} ctas={num_ctas}")


MULTI = [(4, 4, "bf16", 0), (8, 4, "fp16", 0), (1, 16, "bf16", 3), (2, 64, "bf16", 0)]


@pytest.mark.parametrize("G,Lq,dtype,num_ctas", MULTI, ids=[f"G{g}-L{l}-{t}-ctas{n}" for g, l, t, n in MULTI])
def test_multi_rising_scores(cuda_device, G, Lq, dtype, num_ctas):
    """Token-major multi-query tiles (G x q_len rows up to 32, and row tiles
    of 32 beyond)."""
    from test_gpu_multi import _inputs, _oracle, _run

    seed = 8400 + 10 * G + Lq
    L, V0, q0 = _inputs(seed, [n for n in LENS if n >= Lq], G, Lq, dtype)
    V, q = rising_scores(L, V0, q0, seed)
    out, st = _run(cuda_device, L, V, q, num_ctas)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(L, V, q), f"rising multi G={G} q_len={Lq} {dtype}")


@pytest.mark.parametrize("num_ctas", [0, 5])
def test_shared_prefix_rising_scores(cuda_device, num_ctas):
    """Group units: the shared blocks' keys rise with their position like
    every member's own."""
    import paged_kv_cache_357_b200 as pa
    from test_gpu_shared_prefix import _forked_layout, _run

    prompts = [(2048, [1, 100, 513]), (300, [1, 2, 17, 64]), (1000, [3, 40, 200, 7])]
    L = _forked_layout(8500 + num_ctas, prompts, G=8)
    V0 = fill_values_numpy(L)
    V, q = rising_scores(L, V0, V0.q, 8500 + num_ctas)
    V.q = q
    groups = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, 4)
    out, st, _, _ = _run(cuda_device, L, V, groups, 4, num_ctas)
    assert st == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out), ref, f"rising shared prefix ctas={num_ctas}")


def _far_below(layout, values, q_bits, seed):
    """Every key near one shared direction u (entries +-1) and every query
    along -12 u: all scores of a row lie about 200 (log2 units) below 0, far
    under the first chunk's starting reference, with an ordinary spread
    among themselves."""
    from dataclasses import replace

    from pa_testlib import bits_to_f32
    from workloads import f32_to_bits

    dt = layout.dtype
    rng = np.random.default_rng([seed, 9])
    D = layout.head_dim
    u = rng.choice([-1.0, 1.0], size=D).astype(np.float32)
    k = bits_to_f32(values.k_pool, dt)
    finite = np.isfinite(k)
    k = np.where(finite, u + 0.3 * rng.standard_normal(k.shape).astype(np.float32), k)
    q = bits_to_f32(q_bits, dt)
    q = -12.0 * u + 0.3 * rng.standard_normal(q.shape).astype(np.float32)
    nk = values.new_k
    if layout.num_new_tokens > 0:
        nk = f32_to_bits(u + 0.3 * rng.standard_normal(bits_to_f32(nk, dt).shape).astype(np.float32), dt)
    return replace(values, k_pool=f32_to_bits(k, dt), new_k=nk), f32_to_bits(q, dt)


FAR = [(4, 128, "bf16"), (1, 128, "fp16"), (4, 64, "bf16")]


@pytest.mark.parametrize("G,D,dtype", FAR, ids=[f"G{g}-D{d}-{t}" for g, d, t in FAR])
def test_decode_scores_far_below_zero(cuda_device, G, D, dtype):
    """Scores far below 0 on a segment's first chunk (where the tensor-core
    kernels start from reference 0): the rows must move to their exact
    maxima rather than lose every probability to underflow."""
    seed = 8600 + G + D
    L = random_layout(seed, LENS, dtype=dtype, block_size=16, num_q_heads=2 * G, num_kv_heads=2, head_dim=D,
                      write_new_token=True)
    V0 = fill_values_numpy(L)
    V, q = _far_below(L, V0, V0.q, seed)
    V.q = q
    out, st = gpu_step(to_device(L, V, cuda_device), L, num_ctas=37)
    assert int(st.item()) == 0
    ref, _, _ = oracle_step(L, V)
    assert np.abs(ref).max() > 0.05  # the outputs are not all near zero
    assert_attention_close(torch_f64(out), ref, f"far below zero G={G} D={D} {dtype}")


def test_multi_and_prefill_scores_far_below_zero(cuda_device):
    """The same inputs through multi-query tiles (q_len 4) and the
    query-major prefill kernel (q_len 128)."""
    from test_gpu_multi import _inputs, _oracle, _run

    for G, Lq in ((4, 4), (4, 128)):
        seed = 8700 + Lq
        L, V0, q0 = _inputs(seed, [n for n in LENS if n >= Lq], G, Lq, "bf16")
        V, q = _far_below(L, V0, q0, seed)
        out, st = _run(cuda_device, L, V, q, 0)
        assert st == 0
        assert_attention_close(torch_f64(out), _oracle(L, V, q), f"far below zero multi G={G} q_len={Lq}")
