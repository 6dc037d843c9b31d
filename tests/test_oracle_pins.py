"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test ties one part of the oracle to a value the format standard or the mathematics
fixes: the hand-typed OCP MX tables, exact rational arithmetic, brute force, closed forms of
the layer and invariants (sparsity, permutation, scale linearity).  Each is chosen so that a
plausible slip in the oracle (a swapped nibble, a wrong block index, a transposed operand, a
dropped term, a wrong tie-break) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TINY = synth.TINY


def _table(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()
        out[int(a)] = float(b)
    return out


E2M1 = _table("e2m1_ocp_mx_v1.txt")
E8M0 = _table("e8m0_ocp_mx_v1.txt")


# ---- number formats ------------------------------------------------------------------------

def test_e2m1_matches_ocp_table():
    for code, v in E2M1.items():
        got = oracle.e2m1(code)
        assert got == v and math.copysign(1, got) == math.copysign(1, v), code


def test_e2m1_matches_bitfield_definition():
    # sign s, exponent e (2 bits, bias 1), mantissa m (1 bit); e = 0 is subnormal: 0.5 * m
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
        assert oracle.e2m1(code) == (-mag if s else mag)


def test_e8m0_matches_ocp_table():
    for s, v in E8M0.items():
        assert oracle.e8m0(s) == v, s
    assert math.isnan(oracle.e8m0(255))


def test_bf16_decode_matches_ieee_view():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, 4000, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite only
    ref = synth.bf16_to_f32(bits).astype(np.float64)
    got = np.array([oracle.bf16(int(b)) for b in bits])
    assert np.array_equal(got, ref)


def test_mxfp4_nibble_order_and_block_scale():
    # one row of K=64: byte j holds element 2j (low nibble) and 2j+1 (high nibble);
    # elements 0..31 use scale byte 0, 32..63 scale byte 1.
    q = np.zeros((1, 32), dtype=np.uint8)
    q[0, 0] = 0x21      # element 0 = code 1 (0.5), element 1 = code 2 (1.0)
    q[0, 15] = 0x7B     # element 30 = code 0xB (-1.5), element 31 = code 7 (6.0)
    q[0, 16] = 0x0C     # element 32 = code 0xC (-2.0), element 33 = 0
    s = np.array([[127 - 1, 127 + 3]], dtype=np.uint8)  # 0.5, 8
    el = lambda k: oracle.mxfp4_element(q, s, 0, k)
    assert el(0) == 0.25 and el(1) == 0.5
    assert el(30) == -0.75 and el(31) == 3.0
    assert el(32) == -16.0 and el(33) == 0.0


def _decode_reference(q, s):
    """Dense decode of an MXFP4 matrix from the hand-typed tables (test-side, no oracle code)."""
    N, K = q.shape[0], q.shape[1] * 2
    lo = np.vectorize(E2M1.get)(q & 15)
    hi = np.vectorize(E2M1.get)(q >> 4)
    vals = np.empty((N, K))
    vals[:, 0::2] = lo
    vals[:, 1::2] = hi
    scale = np.array([2.0 ** (int(b) - 127) for b in s.ravel()]).reshape(s.shape)
    return vals * np.repeat(scale, 32, axis=1)


def test_mxfp4_exhaustive_bytes_and_scales():
    # every byte value in every position class, under each scale byte of the workload range
    q = np.tile(np.arange(256, dtype=np.uint8), (5, 1))           # [5, 256] -> K = 512
    s = np.repeat(np.arange(121, 126, dtype=np.uint8)[:, None], 16, axis=1)
    ref = _decode_reference(q, s)
    for n in range(5):
        for k in range(512):
            assert oracle.mxfp4_element(q, s, n, k) == ref[n, k]
    # and through the matrix-vector product: one-hot columns pick the decoded column
    for k in (0, 1, 31, 32, 33, 255, 510, 511):
        v = np.zeros(512)
        v[k] = 1.0
        assert np.array_equal(oracle.mxfp4_matvec(q, s, v), ref[:, k])


def test_mxfp4_matvec_random_against_dense_decode():
    rng = np.random.default_rng(1)
    q = rng.integers(0, 256, (40, 96), dtype=np.uint8)
    s = rng.integers(118, 132, (40, 6), dtype=np.uint8)
    v = rng.standard_normal(192)
    ref = _decode_reference(q, s) @ v
    np.testing.assert_allclose(oracle.mxfp4_matvec(q, s, v), ref, rtol=1e-12, atol=1e-12)


def test_bf16_matvec_orientation():
    # W[n][k] = 1 at k = n + 1 (shifted identity): out[n] = v[n+1]; a transposed read gives v[n-1]
    N, K = 8, 12
    W = np.zeros((N, K), dtype=np.uint16)
    for n in range(N):
        W[n, n + 1] = 0x3F80  # 1.0
    v = np.arange(K, dtype=np.float64) + 0.25
    assert np.array_equal(oracle.bf16_matvec(W, v), v[1:N + 1])


# ---- routing ---------------------------------------------------------------------------------

def _bf16_exact(bits):
    return Fraction(float(synth.bf16_to_f32(np.array([bits], dtype=np.uint16))[0]))


def test_router_logits_equal_exact_sum_rounded_once():
    rng = np.random.default_rng(2)
    E, H, B = 6, 32, 3
    R = synth.f32_to_bf16(rng.standard_normal((E, H)).astype(np.float32) * 0.2)
    x = synth.f32_to_bf16(rng.standard_normal((B, H)).astype(np.float32))
    got = oracle.router_logits(R, x)
    for b in range(B):
        for e in range(E):
            exact = sum(_bf16_exact(R[e, j]) * _bf16_exact(x[b, j]) for j in range(H))
            as_double = float(exact)
            assert Fraction(as_double) == exact  # exact in double for this range, so one rounding
            assert got[b, e] == np.float32(as_double)


def test_score_closed_forms():
    assert oracle.score(0.0) == 0.5
    # sigmoid(ln(p/(1-p))) = p for p = 0.75, 0.2, 0.9 (to fp32)
    for p in (0.75, 0.2, 0.9):
        lg = float(np.float32(math.log(p / (1 - p))))
        assert abs(oracle.score(lg) - p) <= 2 ** -23
    assert oracle.score(40.0) == 1.0          # saturates to exactly 1 in fp32
    assert oracle.score(-200.0) == 0.0 or oracle.score(-200.0) < 1e-80
    xs = np.linspace(-20, 20, 2001).astype(np.float32)
    ss = [oracle.score(float(z)) for z in xs]
    assert all(a <= b for a, b in zip(ss, ss[1:]))  # monotone


def test_score_matches_high_precision_sigmoid():
    # 50-digit decimal sigmoid, rounded to double then fp32, on 4000 fp32 logits across the range
    # where the score is neither 0 nor saturated: the fp64 evaluation with libm exp must give the
    # same fp32 bits (it could differ only within ~1e-16 relative of an fp32 rounding boundary)
    from decimal import Decimal, getcontext
    getcontext().prec = 50
    rng = np.random.default_rng(17)
    lg = np.concatenate([rng.normal(0, 3, 3000), rng.uniform(-60, 30, 1000)]).astype(np.float32)
    for v in lg:
        exact = Decimal(1) / (Decimal(1) + (-Decimal(float(v))).exp())
        assert np.float32(float(exact)) == np.float32(oracle.score(float(v))), float(v)


def test_oracle_threads_do_not_change_any_bit(tmp_path):
    # the OpenMP row loops (the timed CPU baseline uses every core) give the same bits as one thread
    import subprocess
    import sys
    w = synth.WORKLOADS["mid_b2"]
    W = synth.layer_weights(w, 0)
    x = synth.tokens(w, batch=5)
    many = oracle.step(w.dims, W, x)
    assert oracle.threads() > 1 or os.cpu_count() == 1
    code = ("import sys, numpy as np; sys.path.insert(0, %r); import oracle, synth; "
            "w = synth.WORKLOADS['mid_b2']; r = oracle.step(w.dims, synth.layer_weights(w, 0), synth.tokens(w, batch=5)); "
            "assert oracle.threads() == 1; np.savez(%r, **r)") % (ROOT, str(tmp_path / "one.npz"))
    env = dict(os.environ, OMP_NUM_THREADS="1")
    subprocess.check_call([sys.executable, "-c", code], env=env)
    one = np.load(tmp_path / "one.npz")
    for k in many:
        assert np.array_equal(many[k], one[k]), k


def _brute_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda e: (-float(scores[e]), e))
    return np.array(order[:k], dtype=np.int32)


@pytest.mark.parametrize("seed", range(5))
def test_topk_matches_brute_force_sort(seed):
    rng = np.random.default_rng(seed)
    s = rng.random(896).astype(np.float32)
    if seed % 2:
        s = np.round(s * 50).astype(np.float32) / 50   # many exact ties
    for k in (1, 4, 16, 896):
        idx, w = oracle.topk(s, k)
        assert np.array_equal(idx, _brute_topk(s, k))
        assert abs(float(w.astype(np.float64).sum()) - 1.0) < 1e-5


def test_topk_ties_lower_index_wins_and_equal_weights():
    s = np.full(64, 0.5, dtype=np.float32)
    s[[3, 9, 40, 41]] = 1.0          # saturated scores tie at 1.0
    idx, w = oracle.topk(s, 4)
    assert list(idx) == [3, 9, 40, 41]
    assert np.all(w == np.float32(0.25))
    idx, w = oracle.topk(s, 6)
    assert list(idx) == [3, 9, 40, 41, 0, 1]
    idx, w = oracle.topk(s, 1)
    assert list(idx) == [3] and w[0] == 1.0


def test_duplicated_router_rows_tie_to_lower_index():
    rng = np.random.default_rng(3)
    E, H = 64, 512
    R = synth.f32_to_bf16((rng.standard_normal((E, H)) / math.sqrt(H)).astype(np.float32))
    x = synth.f32_to_bf16(rng.standard_normal((1, H)).astype(np.float32))
    logits, _, _ = oracle.route(R, x, 4)
    top = int(np.argmax(logits[0]))
    R2 = R.copy()
    R2[top + 1 if top + 1 < E else top - 1] = R[top]
    lo, hi = sorted((top, top + 1 if top + 1 < E else top - 1))
    _, idx, w = oracle.route(R2, x, 4)
    assert idx[0, 0] == lo and idx[0, 1] == hi and w[0, 0] == w[0, 1]


# ---- the step: closed forms and invariants on the tiny layer --------------------------------

@pytest.fixture(scope="module")
def tiny():
    w = synth.WORKLOADS["tiny_b1"]
    W = synth.layer_weights(w, 0)
    x = synth.tokens(w, batch=3)
    return W, x


def _copy(W):
    return {k: v.copy() for k, v in W.items()}


def test_dense_masked_equals_sparse_bitwise(tiny):
    W, x = tiny
    a = oracle.step(TINY, W, x)
    b = oracle.step(TINY, W, x, dense_masked=True)
    for key in ("out", "ylat", "h", "sh"):
        assert np.array_equal(a[key], b[key]), key


def test_latent_projection_is_wdn_times_x(tiny):
    W, x = tiny
    W2 = _copy(W)
    W2["w_down_lat"][:] = 0
    for l in range(TINY.latent):
        W2["w_down_lat"][l, l + 1] = 0x3F80      # h[l] = x[l+1]
    r = oracle.step(TINY, W2, x)
    assert np.array_equal(r["h"], synth.bf16_to_f32(x[:, 1:TINY.latent + 1]).astype(np.float64))


def test_silu_zero_gate_leaves_shared_only(tiny):
    W, x = tiny
    W2 = _copy(W)
    W2["gate_q"][:] = 0
    r = oracle.step(TINY, W2, x)
    assert np.all(r["ylat"] == 0) and np.array_equal(r["out"], r["sh"])


def test_zero_up_projection_leaves_shared_only(tiny):
    W, x = tiny
    W2 = _copy(W)
    W2["w_up_lat"][:] = 0
    r = oracle.step(TINY, W2, x)
    assert np.array_equal(r["out"], r["sh"])


def test_zero_shared_codes_leave_routed_only(tiny):
    W, x = tiny
    W2 = _copy(W)
    for n in ("sh_gate_q", "sh_up_q", "sh_down_q"):
        W2[n][:] = 0
    r = oracle.step(TINY, W2, x)
    assert np.all(r["sh"] == 0)
    up = np.stack([oracle.bf16_matvec(W["w_up_lat"], r["ylat"][b]) for b in range(x.shape[0])])
    assert np.array_equal(r["out"], up)


def test_all_ones_experts_closed_form(tiny):
    # every gate/up/down element = 1.0 (code 2, scale 127): g = u = sum(h) on every row,
    # a = silu(sum h) * sum h, y = I * a on every latent row, ylat = (sum w) * I * a
    W, x = tiny
    W2 = _copy(W)
    for n in ("gate_q", "up_q", "down_q"):
        W2[n][:] = 0x22
    for n in ("gate_s", "up_s", "down_s"):
        W2[n][:] = 127
    r = oracle.step(TINY, W2, x)
    for b in range(x.shape[0]):
        sh_ = r["h"][b].sum()
        a = sh_ / (1 + math.exp(-sh_)) * sh_
        expect = float(r["w"][b].astype(np.float64).sum()) * TINY.expert_inter * a
        np.testing.assert_allclose(r["ylat"][b], expect, rtol=1e-12)


def test_one_hot_expert_orientation(tiny):
    # expert e has a single nonzero gate element 1.0 and up element 2.0 at (i0, l0) and a down
    # element 1.0 at (l1, i0): y_e[l1] = silu(h[l0]) * 2 h[l0] (gate inside silu, up outside),
    # all other y_e entries 0.
    W, x = tiny
    r0 = oracle.step(TINY, W, x[:1])
    e = int(r0["idx"][0, 0])
    i0, l0, l1 = 5, 77, 130
    W2 = _copy(W)
    for n in ("gate_q", "up_q", "down_q"):
        W2[n][e] = 0
    for n in ("gate_s", "up_s", "down_s"):
        W2[n][e] = 127
    W2["gate_q"][e, i0, l0 // 2] = 0x02 if l0 % 2 == 0 else 0x20
    W2["up_q"][e, i0, l0 // 2] = 0x04 if l0 % 2 == 0 else 0x40
    W2["down_q"][e, l1, i0 // 2] = 0x02 if i0 % 2 == 0 else 0x20
    h = r0["h"][0]
    y = oracle.expert(TINY, W2, e, h)
    expect = np.zeros(TINY.latent)
    expect[l1] = h[l0] / (1 + math.exp(-h[l0])) * (2 * h[l0])
    assert np.array_equal(y, expect)


def test_one_hot_shared_expert_orientation(tiny):
    # shared gate element 1.0 and up element -3.0 at (i0, j0), down element 0.5 at (j1, i0):
    # sh[j1] = 0.5 * silu(x[j0]) * (-3 x[j0]); every other entry 0.
    W, x = tiny
    H = TINY.hidden
    i0, j0, j1 = 9, 301, 44
    W2 = _copy(W)
    for n in ("sh_gate_q", "sh_up_q", "sh_down_q"):
        W2[n][:] = 0
    for n in ("sh_gate_s", "sh_up_s", "sh_down_s"):
        W2[n][:] = 127
    W2["sh_gate_q"][i0, j0 // 2] = 0x02 if j0 % 2 == 0 else 0x20
    W2["sh_up_q"][i0, j0 // 2] = 0x0D if j0 % 2 == 0 else 0xD0
    W2["sh_down_q"][j1, i0 // 2] = 0x01 if i0 % 2 == 0 else 0x10
    xd = synth.bf16_to_f32(x[0]).astype(np.float64)
    sh = oracle.shared_expert(TINY, W2, xd)
    expect = np.zeros(H)
    expect[j1] = 0.5 * (xd[j0] / (1 + math.exp(-xd[j0]))) * (-3 * xd[j0])
    assert np.array_equal(sh, expect)


def test_down_scale_doubling_doubles_latent_sum(tiny):
    W, x = tiny
    W2 = _copy(W)
    W2["down_s"] += 1
    a, b = oracle.step(TINY, W, x), oracle.step(TINY, W2, x)
    assert np.array_equal(b["ylat"], 2 * a["ylat"])
    assert np.array_equal(a["idx"], b["idx"])


def test_unselected_expert_weights_do_not_matter(tiny):
    W, x = tiny
    r = oracle.step(TINY, W, x)
    unused = sorted(set(range(TINY.n_experts)) - set(r["idx"].ravel().tolist()))[:5]
    W2 = _copy(W)
    for e in unused:
        for n in ("gate_q", "up_q", "down_q"):
            W2[n][e] = 0x77
    r2 = oracle.step(TINY, W2, x)
    assert np.array_equal(r["out"], r2["out"])


def test_expert_permutation_invariance(tiny):
    W, x = tiny
    rng = np.random.default_rng(4)
    perm = rng.permutation(TINY.n_experts)          # new expert p holds old expert perm[p]
    W2 = _copy(W)
    W2["router"] = W["router"][perm].copy()
    for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s"):
        W2[n] = W[n][perm].copy()
    a, b = oracle.step(TINY, W, x), oracle.step(TINY, W2, x)
    assert np.array_equal(perm[b["idx"]], a["idx"])
    np.testing.assert_allclose(b["out"], a["out"], rtol=1e-12, atol=1e-9)


def test_tokens_are_independent(tiny):
    W, x = tiny
    full = oracle.step(TINY, W, x)
    one = oracle.step(TINY, W, x, tokens=range(1, 2))
    for key in ("out", "h", "ylat", "sh", "logits", "idx", "w"):
        assert np.array_equal(one[key][0], full[key][1]), key


def test_full_size_b2_tokens_share_some_experts():
    w = synth.WORKLOADS["full_b2"]
    R = synth.router_weights(w, 0)
    _, idx, _ = oracle.route(R, synth.tokens(w), w.dims.top_k)
    common = len(set(idx[0].tolist()) & set(idx[1].tolist()))
    assert 0 < common < w.dims.top_k
