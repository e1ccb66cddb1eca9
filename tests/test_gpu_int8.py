"""GPU parity of the INT8 query/key path: fh_quantize_int8_rows (bit-exact with
the oracle's per-row symmetric quantization) and fh_int8_attention_scores
(within the oracle's tolerance for three FP32 roundings of an exact product).

FastH3 Trim (comfyui-wiki news), "How fast it runs": the query and the key are
quantized to INT8 for the attention scores."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _gpu_util import fh, to_dev

pytestmark = pytest.mark.gpu


def _gpu_quantize_rows(x_bits: np.ndarray, ldx: int | None = None):
    m = fh()
    rows, d = x_bits.shape
    x = to_dev(x_bits, ldx)
    q = torch.full((rows, d), 0x55, dtype=torch.int8, device="cuda")
    s = torch.full((rows,), float("nan"), dtype=torch.float32, device="cuda")
    m.fh_quantize_int8_rows(x, q, s)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


def _assert_rows_exact(x_bits, ldx=None):
    q, s = _gpu_quantize_rows(x_bits, ldx)
    rq, rs = oracle.quantize_int8_rows(x_bits)
    np.testing.assert_array_equal(s.view(np.uint32), rs.view(np.uint32))
    bad = np.argwhere(q != rq)
    assert bad.size == 0, f"{len(bad)} INT8 codes differ, first at {bad[:5].tolist()}"


# One case per launch form of the row quantizer (lanes per row x chunks per
# lane: 4x1, 8x1, 16x1, 32x1, 32x2, 32x4, 32x8, and the general two-pass form),
# ragged row counts, a row stride wider than d, and a size that needs the
# grid-stride loop.
@pytest.mark.parametrize("rows,d,ldx", [(1, 8, None), (77, 40, 48), (1000, 64, 72), (300, 128, None),
                                        (257, 136, None), (3, 200, None), (20, 384, None), (130, 520, 528),
                                        (9, 1024, None), (17, 2048, None), (33, 2688, None), (200000, 32, None)])
def test_quantize_rows_bit_exact(rows, d, ldx):
    x = S.attention_qk(1, rows, d, "rows", seed=rows + d).reshape(rows, d)
    _assert_rows_exact(x, ldx)


def test_quantize_rows_edge_values():
    """Zero rows, a row whose amax is negative, half-way quotients, a row so
    small that its scale is subnormal in FP32, and a row of huge values."""
    d = 64
    x = np.zeros((6, d))
    x[1, :] = np.linspace(-3.0, 2.0, d)                      # amax from a negative value
    x[2, :8] = [127.0, 0.5, 1.5, 2.5, -0.5, -1.5, 126.5, -126.5]  # s = 1: ties to even
    x[3, :] = np.linspace(-1.0, 1.0, d) * 1e-38              # subnormal scale
    x[4, :] = np.linspace(-1.0, 1.0, d) * 3e38               # near the top of the range
    x[5, 5] = -7.0                                           # one non-zero element
    _assert_rows_exact(S.to_bf16_bits(x))


def _scores_case(H, tq, tk, d, seed=0, zero_rows=()):
    """GPU quantization of seeded Q and K, checked bit-exact, then GPU scores."""
    m = fh()
    qb = S.attention_qk(H, tq, d, "q", seed)
    kb = S.attention_qk(H, tk, d, "k", seed)
    for h, i in zero_rows:
        qb[h, i, :] = 0
    q8, qs = _gpu_quantize_rows(qb.reshape(H * tq, d))
    k8, ks = _gpu_quantize_rows(kb.reshape(H * tk, d))
    rq8, rqs = oracle.quantize_int8_rows(qb.reshape(H * tq, d))
    rk8, rks = oracle.quantize_int8_rows(kb.reshape(H * tk, d))
    assert np.array_equal(q8, rq8) and np.array_equal(qs.view(np.uint32), rqs.view(np.uint32))
    assert np.array_equal(k8, rk8) and np.array_equal(ks.view(np.uint32), rks.view(np.uint32))
    sm_scale = float(np.float32(1.0 / math.sqrt(d)))
    # Output inside a poisoned buffer with a guard region after it.
    n = H * tq * tk
    buf = torch.full((n + 256,), float("nan"), dtype=torch.float32, device="cuda")
    buf[n:] = 12345.0
    out = buf[:n].view(H, tq, tk)
    m.fh_int8_attention_scores(torch.from_numpy(q8).cuda().view(H, tq, d), torch.from_numpy(qs).cuda(),
                               torch.from_numpy(k8).cuda().view(H, tk, d), torch.from_numpy(ks).cuda(),
                               sm_scale, out)
    torch.cuda.synchronize()
    m.fh_device_status()
    assert (buf[n:] == 12345.0).all(), "the score kernel wrote past the end of S"
    return (q8.reshape(H, tq, d), qs.reshape(H, tq), k8.reshape(H, tk, d), ks.reshape(H, tk), sm_scale,
            out.cpu().numpy())


def _assert_scores(s, ref):
    tol = oracle.int8_scores_tolerance(ref)
    err = np.abs(s.astype(np.float64) - ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{len(bad)} scores out of tolerance, first at {bad[:5].tolist()}: "
                           f"{s[tuple(bad[0])]} vs {ref[tuple(bad[0])]}")


@pytest.mark.parametrize("H,tq,tk,d", [(1, 1, 4, 16), (3, 200, 300, 128), (2, 130, 516, 256), (2, 257, 260, 64),
                                       (1, 128, 256, 144), (4, 333, 1000, 128), (1, 600, 4, 32),
                                       (2, 77, 301, 128), (1, 5, 1, 16), (3, 129, 258, 64)])
def test_scores_match_oracle(H, tq, tk, d):
    q8, qs, k8, ks, sm_scale, s = _scores_case(H, tq, tk, d, seed=tq)
    _assert_scores(s, oracle.int8_scores(q8, qs, k8, ks, sm_scale))


def test_scores_zero_query_rows_are_zero():
    q8, qs, k8, ks, sm_scale, s = _scores_case(2, 150, 280, 128, seed=7, zero_rows=((0, 3), (1, 149)))
    assert qs[0, 3] == 0 and qs[1, 149] == 0
    assert (s[0, 3] == 0).all() and (s[1, 149] == 0).all()
    _assert_scores(s, oracle.int8_scores(q8, qs, k8, ks, sm_scale))


def test_scores_extreme_codes_exact_accumulation():
    """All codes +-127 with d = 2688: |acc| reaches 127^2 * 2688 = 43,354,752 > 2^24,
    so the INT32 sum must be exact on the tensor cores and only its conversion rounds."""
    m = fh()
    H, tq, tk, d = 1, 130, 260, 2688
    sign_q = np.where(S.u64(S.derive_seed("ext", "q"), 0, tq * d) % 2 == 0, 1, -1).reshape(H, tq, d)
    sign_k = np.where(S.u64(S.derive_seed("ext", "k"), 0, tk * d) % 2 == 0, 1, -1).reshape(H, tk, d)
    sign_k[0, 0] = sign_q[0, 0]  # one score at the full +127^2 d
    q8 = (127 * sign_q).astype(np.int8)
    k8 = (127 * sign_k).astype(np.int8)
    qs = np.full((H, tq), np.float32(0.01), dtype=np.float32)
    ks = np.full((H, tk), np.float32(0.02), dtype=np.float32)
    out = torch.full((H, tq, tk), float("nan"), dtype=torch.float32, device="cuda")
    m.fh_int8_attention_scores(torch.from_numpy(q8).cuda(), torch.from_numpy(qs).cuda(), torch.from_numpy(k8).cuda(),
                               torch.from_numpy(ks).cuda(), 1.0, out)
    torch.cuda.synchronize()
    m.fh_device_status()
    s = out.cpu().numpy()
    ref = oracle.int8_scores(q8, qs, k8, ks, 1.0)
    _assert_scores(s, ref)


def test_scores_full_size_sampled():
    """21 heads x 4096 queries x 4096 keys x d 128 (the launch the benchmark
    times): every code and scale bit-exact, scores of 96 sampled query rows
    (each against all keys) within tolerance, and every score finite."""
    H, T, d = 21, 4096, 128
    q8, qs, k8, ks, sm_scale, s = _scores_case(H, T, T, d, seed=1)
    assert np.isfinite(s).all()
    pick = S.u64(S.derive_seed("int8-full", "rows"), 0, 96) % np.uint64(H * T)
    for flat in pick.tolist():
        h, i = divmod(int(flat), T)
        ref = oracle.int8_scores(q8[h:h + 1, i:i + 1], qs[h:h + 1, i:i + 1], k8[h:h + 1], ks[h:h + 1], sm_scale)
        _assert_scores(s[h:h + 1, i:i + 1], ref)


def test_score_stall_times_out_drains_and_context_survives(monkeypatch):
    """With the test hook FH_INT8_TEST_STALL=1 the first CTA's MMA warp stops
    before its first MMA without committing; that CTA's producer and epilogue
    run into their bounded waits (about 4 s), drain and free TMEM, and the host
    reads FH_ERR_TIMEOUT.  With the hook off, scores in the same context pass."""
    m = fh()
    m.fh_device_status()
    H, T, d = 2, 300, 128
    q8 = torch.zeros((H, T, d), dtype=torch.int8, device="cuda")
    qs = torch.ones((H, T), dtype=torch.float32, device="cuda")
    s = torch.empty((H, T, T), dtype=torch.float32, device="cuda")
    monkeypatch.setenv("FH_INT8_TEST_STALL", "1")
    m.fh_int8_attention_scores(q8, qs, q8, qs, 1.0, s)
    with pytest.raises(m.FHError) as e:
        m.fh_device_status()
    assert e.value.status == m.FH_ERR_TIMEOUT
    monkeypatch.delenv("FH_INT8_TEST_STALL")
    m.fh_device_status()  # the word was cleared
    q8a, qsa, k8a, ksa, sm_scale, sa = _scores_case(2, 300, 260, 128, seed=11)
    _assert_scores(sa, oracle.int8_scores(q8a, qsa, k8a, ksa, sm_scale))
