"""CPU checks of the arithmetic the tensor-core e4m3 decode kernel uses
(decode_tc8.cuh), simulated in float64 with the oracle's e4m3 rounding: its
e4m3 MMAs take e4m3 operands on both sides, so q and the softmax weights P
enter as sums of e4m3 terms, term i+1 carrying 16x the rounding residual of
term i.  These tests fix how many terms each side needs: q three (every f16 q
held to 2^-24 of its head's largest element), P four (three miss the output
tolerance over full-range codes).  The pools' cache format is the overview
page's FP8 KV cache (§5.1); the attention is the paging page's §3 phase 2."""
import numpy as np

from oracle import fp8

TOL = 2e-3  # the 16-bit decode tolerance: |err| <= TOL * max(1, |ref|)


def _e4m3(x):
    return fp8.e4m3_decode(fp8.e4m3_encode(np.asarray(x, np.float32))).astype(np.float64)


def _terms(x, n):
    out, r = [], np.asarray(x, np.float64)
    for _ in range(n):
        t = _e4m3(r.astype(np.float32))
        out.append(t)
        r = (r - t) * 16.0
    return out


def _q_scale(q):
    """The kernel's per-head power of two c: max|q| * c in [128, 256)."""
    mx = float(np.max(np.abs(q)))
    return 2.0 ** (7 - int(np.floor(np.log2(mx)))) if mx > 0 else 128.0


def test_three_e4m3_terms_hold_f16_q():
    rng = np.random.default_rng(11)
    worst = 0.0
    for _ in range(300):
        mag = 2.0 ** float(rng.integers(-20, 14))
        q = (rng.standard_normal(128) * mag).astype(np.float16)
        q[rng.integers(0, 128, 4)] = (rng.standard_normal(4) * mag * 2.0 ** float(rng.integers(-12, 0))).astype(np.float16)
        x = q.astype(np.float64) * _q_scale(q)
        got = sum(t / 16.0 ** i for i, t in enumerate(_terms(x, 3)))
        assert np.max(np.abs(x)) < 256.0  # no term saturates (e4m3 max 448)
        worst = max(worst, float(np.max(np.abs(got - x)) / np.max(np.abs(x))))
    assert worst < 2.0 ** -24
    # two terms are not enough (an f16 has 11 significant bits, a term 4):
    # 1 + 2^-1 + 2^-5 + 2^-10 scaled by 128 is 196.125 = 192 + 64/16 + 32/256
    x = np.array([np.float16(1.5322265625)], np.float64) * 128
    assert [float(t[0]) for t in _terms(x, 3)] == [192.0, 64.0, 32.0]
    two = sum(t / 16.0 ** i for i, t in enumerate(_terms(x, 2)))
    assert two[0] == 196.0 != x[0]


def _codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 1  # no NaN codes
    return c


def _kernel_sim(q, kc, vc, scale, k_scale, v_scale, p_terms, chunk=128, thr=8.0):
    """One (sequence, head) of the tensor-core kernel in float64: S from three
    q terms, the running max moved only past 2^thr, P as p_terms e4m3 terms."""
    K = fp8.e4m3_decode(kc).astype(np.float64)
    V = fp8.e4m3_decode(vc).astype(np.float64)
    qf = q.astype(np.float32)
    c = _q_scale(qf)
    cols = [K @ t for t in _terms(qf.astype(np.float64) * c, 3)]
    s = (cols[0] + cols[1] / 16 + cols[2] / 256) / c * scale * k_scale * np.log2(np.e)
    s = s.astype(np.float32).astype(np.float64)
    m, l, o = -np.inf, 0.0, np.zeros(V.shape[1])
    for a in range(0, len(s), chunk):
        mc = s[a:a + chunk].max()
        if mc > m + thr:
            f = 0.0 if m == -np.inf else 2.0 ** (m - mc)
            o, l, m = o * f, l * f, mc
        p = np.exp2(s[a:a + chunk] - m).astype(np.float32)
        assert p.max() <= 2.0 ** thr <= 448
        l += float(p.astype(np.float64).sum())
        o += sum((t @ V[a:a + chunk]) / 16.0 ** i for i, t in enumerate(_terms(p, p_terms)))
    return v_scale * o / l


def test_four_p_terms_meet_the_tolerance_and_three_do_not():
    worst = {3: 0.0, 4: 0.0}
    for k_scale, v_scale, seed in [(0.25, 0.5, 5), (2.0, 0.125, 6), (0.0625, 0.5, 7)]:
        rng = np.random.default_rng(seed)
        for _ in range(40):
            L = int(rng.integers(1, 2000))
            kc, vc = _codes(rng, (1, 1, L, 128)), _codes(rng, (1, 1, L, 128))
            q = rng.standard_normal((1, 1, 128)).astype(np.float16)
            scale = 1 / np.sqrt(128)
            ref = fp8.paged_decode_attention_fp8(q, kc, vc, np.zeros((1, 1), np.int32), np.array([L]), scale,
                                                 k_scale, v_scale)[0, 0]
            tol = TOL * np.maximum(1.0, np.abs(ref))
            for n in worst:
                got = _kernel_sim(q[0, 0], kc[0, 0], vc[0, 0], scale, k_scale, v_scale, n)
                worst[n] = max(worst[n], float(np.max(np.abs(got - ref) / tol)))
    assert worst[4] < 0.5, worst
    assert worst[3] > 1.0, worst  # three terms of P (12 bits) miss the tolerance
